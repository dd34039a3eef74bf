"""Backward parity: dQ, dK, dV from the CUDA kernels against the float64 oracle.

The GPU backward consumes the GPU forward's O and LSE (the real pipeline); the
oracle recomputes everything from the inputs.  Bound: relative L2 error
<= 2e-2 per gradient tensor.  Dropout keep bits used by the backward kernel are
read back exactly through one-hot dO rows.
"""

import numpy as np
import pytest

from oracle import attention_backward, dropout_keep, dropout_scale
from io_aware_exact_20_b200.workloads import make_block_mask, make_qkvdo, make_seqlens

pytestmark = pytest.mark.gpu

REL_L2 = 2e-2


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def rel_l2(a, ref):
    n = np.linalg.norm(ref)
    return np.linalg.norm(a - ref) / n if n > 0 else np.linalg.norm(a)


def run_bwd(fa, B, H, N, d, causal=False, lens=None, density=None, p=0.0, seed=21, data_seed=3):
    import torch
    q, k, v, do = make_qkvdo(B, H, N, d, data_seed)
    seqlens = None if lens is None else make_seqlens(B, lens[0], lens[1], data_seed + 1)
    bm = None if density is None else make_block_mask(N, density, data_seed + 2)
    scale = d ** -0.5
    gq, gk, gv, gdo = (x.cuda() for x in (q, k, v, do))
    kw = dict(scale=scale, causal=causal, seqlens=seqlens, dropout_p=p, seed=seed, block_mask=bm)
    o, lse = fa.forward(gq, gk, gv, **kw)
    dq, dk, dv = fa.backward(gq, gk, gv, o, lse, gdo, **kw)
    torch.cuda.synchronize()
    assert fa.last_device_status() == 0
    ref = attention_backward(f64(q), f64(k), f64(v), f64(do), scale, causal, seqlens, p, seed, bm)
    return (f64(dq), f64(dk), f64(dv)), ref


CASES = [
    # B, H, N, d, causal, key lengths, block density, dropout p
    (1, 2, 128, 64, False, None, None, 0.0),       # the tiny exact workload
    (1, 1, 1, 64, False, None, None, 0.0),
    (1, 1, 129, 128, True, None, None, 0.0),
    (2, 3, 300, 64, True, None, None, 0.0),
    (2, 2, 384, 128, False, None, None, 0.0),
    (2, 2, 520, 128, True, None, None, 0.0),
    (3, 2, 400, 64, False, (1, 400), None, 0.0),
    (2, 2, 333, 64, True, (0, 60), None, 0.0),     # empty rows and dead key tiles
    (1, 2, 1024, 64, False, None, 0.25, 0.0),
    (1, 2, 640, 128, True, (300, 640), 0.5, 0.0),
    (2, 2, 256, 64, True, None, None, 0.1),
    (2, 2, 384, 128, False, (100, 384), None, 0.2),
    (1, 3, 700, 64, True, (500, 700), 0.4, 0.3),
    # the 256-wide backward (two CTAs per key tile, each with half the columns)
    (1, 2, 128, 256, False, None, None, 0.0),
    (2, 2, 300, 256, True, None, None, 0.1),
    (1, 2, 1000, 192, True, (300, 1000), 0.5, 0.0),
    (2, 1, 777, 256, False, (100, 777), 0.4, 0.2),
]


@pytest.mark.parametrize("B,H,N,d,causal,lens,density,p", CASES)
def test_backward_matches_oracle(lib, parity_record, B, H, N, d, causal, lens, density, p):
    got, ref = run_bwd(lib, B, H, N, d, causal, lens, density, p)
    errs = {}
    for name, a, r in zip(("dq", "dk", "dv"), got, ref):
        assert np.isfinite(a).all(), name
        errs[name] = e = rel_l2(a, r)
        assert e <= REL_L2, (name, e)
    parity_record(**{f"{k}_rel_l2": float(v) for k, v in errs.items()})


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("p", [0.0, 0.1])
def test_backward_block_mask_without_diagonal(lib, parity_record, d, causal, p):
    """Block mask with holes in its diagonal, an all-zero block row (query
    tile 1: rows without keys, so dQ = 0 there) and an all-zero block column
    (key tile 2: reached by no query tile, so dK = dV = 0 there)."""
    import torch
    from test_gpu_fwd import block_mask_with_holes
    B, H, N = 2, 2, 600
    q, k, v, do = make_qkvdo(B, H, N, d, 33)
    bm = block_mask_with_holes(N, 32)
    scale = d ** -0.5
    kw = dict(scale=scale, causal=causal, dropout_p=p, seed=6, block_mask=bm)
    gq, gk, gv, gdo = (x.cuda() for x in (q, k, v, do))
    o, lse = lib.forward(gq, gk, gv, **kw)
    dq, dk, dv = lib.backward(gq, gk, gv, o, lse, gdo, **kw)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    ref = attention_backward(f64(q), f64(k), f64(v), f64(do), scale, causal, None, p, 6, bm)
    got = (f64(dq), f64(dk), f64(dv))
    errs = {}
    for name, a, r in zip(("dq", "dk", "dv"), got, ref):
        assert np.isfinite(a).all(), name
        errs[name] = e = rel_l2(a, r)
        assert e <= REL_L2, (name, e)
    parity_record(**{f"{k}_rel_l2": float(v) for k, v in errs.items()})
    assert (got[0][:, :, 128:256] == 0).all()                          # empty query rows
    assert (got[1][:, :, 256:384] == 0).all() and (got[2][:, :, 256:384] == 0).all()


@pytest.mark.parametrize("d", [64, 256])
def test_backward_is_repeatable_for_dk_dv(lib, d):
    """dK and dV involve no atomics: two runs give identical bits."""
    import torch
    q, k, v, do = (x.cuda() for x in make_qkvdo(1, 2, 512, d, 9))
    o, lse = lib.forward(q, k, v, causal=True, dropout_p=0.1, seed=3)
    a = lib.backward(q, k, v, o, lse, do, causal=True, dropout_p=0.1, seed=3)
    b = lib.backward(q, k, v, o, lse, do, causal=True, dropout_p=0.1, seed=3)
    torch.cuda.synchronize()
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert (a[0].float() - b[0].float()).abs().max().item() < 1e-2


@pytest.mark.parametrize("d", [64, 128, 256])
def test_backward_kernel_dropout_bits_exact(lib, d):
    """Q = 0 gives P = 1/N; dO rows one-hot over a window of d queries give
    dV[j, c] = keep(i0 + c, j) / (N q), q the keep probability: every keep bit the backward
    kernel used for dV is read back and compared with the oracle's."""
    import torch
    B, H, N, p, seed = 1, 2, 256, 0.1, 0x5EED0003
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    gen = torch.Generator().manual_seed(1)
    k = torch.randn(B, H, N, d, generator=gen).to(torch.bfloat16).cuda()
    v = torch.randn(B, H, N, d, generator=gen).to(torch.bfloat16).cuda()
    o, lse = lib.forward(q, k, v, dropout_p=p, seed=seed)
    level = dropout_scale(p) / N
    for i0 in range(0, N, d):
        do = torch.zeros(B, H, N, d, dtype=torch.bfloat16)
        for c in range(d):
            do[:, :, i0 + c, c] = 1.0
        _, _, dv = lib.backward(q, k, v, o, lse, do.cuda(), dropout_p=p, seed=seed)
        dvh = f64(dv)
        got = dvh > 0.5 * level
        for b in range(B):
            for h in range(H):
                keep = dropout_keep(seed, p, b, h, np.arange(N), N)  # [query, key]
                want = keep[i0:i0 + d, :].T                           # [key, c]
                assert np.array_equal(got[b, h], want)
        assert np.abs(dvh[got] - level).max() < 0.01 * level
