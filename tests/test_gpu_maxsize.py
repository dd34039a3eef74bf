"""Parity where the tensors are larger than 2^31 elements: B=1, H=40,
N=2^20, d=64 puts 2.68e9 elements in each of Q, K, V, O, dO, dQ, dK, dV
(5.4 GB each, about 54 GB on the device with the backward workspace), so
that every head from 32 on starts past element 2^31 and every offset the
kernels form (tensor rows, LSE and workspace rows, dQ accumulators, the
dropout counters of rows up to 2^20) must be 64-bit clean.

A block mask that keeps only the diagonal 128 x 128 blocks keeps the work
small (each query tile meets its own key tile) and makes sampled tiles exact
oracle problems of their own: the oracle runs on a tile's 128 rows of Q, K,
V, dO, told the tile's position in the sequence so that dropout draws the
bits of the absolute (b, h, i, j).  Bounds as in the other parity tests."""

import numpy as np
import pytest

from oracle import head_backward_cols, head_backward_rows, head_forward_rows

pytestmark = pytest.mark.gpu

B, H, N, D = 1, 40, 1 << 20, 64
P, SEED = 0.1, 7
# (head, query / key tile): heads on both sides of element 2^31 (head 32 starts there)
SAMPLES = ((0, 0), (31, 3000), (32, 0), (32, 5555), (39, 4097), (39, N // 128 - 1))


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def rel_l2(a, r):
    return np.linalg.norm(a - r) / np.linalg.norm(r)


def test_offsets_past_two_to_the_31_elements(lib):
    import torch
    free, _ = torch.cuda.mem_get_info()
    if free < 64e9:
        pytest.skip(f"needs about 60 GB of free device memory, {free / 1e9:.1f} GB free")
    g = torch.Generator(device="cuda")
    g.manual_seed(2024)
    q, k, v, do = (torch.randn((B, H, N, D), device="cuda", dtype=torch.bfloat16, generator=g)
                   for _ in range(4))
    assert q.numel() > 2 ** 31 and 32 * N * D == 2 ** 31
    scale = D ** -0.5
    kw = dict(scale=scale, causal=False, dropout_p=P, seed=SEED,
              block_mask=np.eye(N // 128, dtype=np.uint8))
    o, lse = lib.forward(q, k, v, **kw)
    dq, dk, dv = lib.backward(q, k, v, o, lse, do, **kw)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    # every row meets its own diagonal block: no empty row anywhere
    assert bool(torch.isfinite(lse).all()) and bool(torch.isfinite(o.float()).all())
    for t in (dq, dk, dv):
        assert bool(torch.isfinite(t.float()).all())

    rows = np.array([0, 1, 64, 126, 127])
    cols = np.array([0, 31, 100, 127])
    okw = dict(dropout_p=P, seed=SEED, b=0)
    for h, t in SAMPLES:
        sl = slice(128 * t, 128 * t + 128)
        qh, kh, vh, doh = (f64(x[0, h, sl]) for x in (q, k, v, do))
        pos = dict(h=h, row0=128 * t, key0=128 * t, **okw)
        ro, rl = head_forward_rows(qh, kh, vh, scale, rows, **pos)
        go = f64(o[0, h, sl])[rows]
        gl = lse[0, h, sl].cpu().numpy().astype(np.float64)[rows]
        assert np.all(np.abs(go - ro) <= 1e-2 + 2.0 ** -8 * np.abs(ro)), (h, t)
        assert np.abs(gl - rl).max() <= 1e-3, (h, t)
        rdq = head_backward_rows(qh, kh, vh, doh, scale, rows, **pos)
        assert rel_l2(f64(dq[0, h, sl])[rows], rdq) <= 2e-2, (h, t)
        rdk, rdv = head_backward_cols(qh, kh, vh, doh, scale, cols, **pos)
        assert rel_l2(f64(dk[0, h, sl])[cols], rdk) <= 2e-2, (h, t)
        assert rel_l2(f64(dv[0, h, sl])[cols], rdv) <= 2e-2, (h, t)
