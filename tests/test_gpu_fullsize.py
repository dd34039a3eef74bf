"""Parity at the full workload sizes, in the launch configuration bench.py
times (same workloads, same seeds, same entry points), on outputs the oracle
can compute one by one: sampled query rows of O, LSE and dQ, sampled key
columns of dK and dV, and, for the 64K block-sparse case, the identity
sum_j dK_j = 0 of every head (the rows of dS sum to zero).

Bounds as in the small-size tests: O within 1e-2 + 2^-8 |O| (bf16 storage),
LSE within 1e-3, dQ / dK / dV relative L2 within 2e-2 over the samples.
"""

import numpy as np
import pytest

from oracle import head_backward_cols, head_backward_rows, head_forward_rows
from io_aware_exact_20_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def sample_rows(N, rng, extra=12):
    fixed = [0, 1, 127, 128, 129, 255, 256, N // 2, N - 129, N - 128, N - 2, N - 1]
    rnd = rng.choice(N, size=min(extra, N), replace=False)
    return np.unique(np.clip(np.concatenate([fixed, rnd]), 0, N - 1))


def rel_l2(a, r):
    n = np.linalg.norm(r)
    return np.linalg.norm(a - r) / n if n > 0 else np.linalg.norm(a)


_CACHE = {}


def run_workload(fa, name):
    """One forward + backward of the whole workload on the GPU (cached)."""
    if name in _CACHE:
        return _CACHE[name]
    import torch
    w = WORKLOADS[name]
    inp = make_inputs(w)
    q, k, v, do = (inp[x].cuda() for x in ("q", "k", "v", "do"))
    kw = dict(scale=w.scale, causal=w.causal, seqlens=inp["seqlens"], dropout_p=w.dropout_p,
              seed=w.dropout_seed, block_mask=inp["block_mask"])
    o, lse = fa.forward(q, k, v, **kw)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, **kw)
    torch.cuda.synchronize()
    assert fa.last_device_status() == 0
    res = (w, inp, o, lse, dq, dk, dv)
    _CACHE[name] = res
    return res


def head_arrays(inp, b, h):
    return tuple(f64(inp[x][b, h]) for x in ("q", "k", "v", "do"))


NAMES = ["gpt2", "bert", "long64", "long128", "sparse"]


@pytest.mark.parametrize("name", NAMES)
def test_fullsize_forward_rows(lib, name):
    w, inp, o, lse, *_ = run_workload(lib, name)
    B, H, N = w.B, w.H, w.N
    rng = np.random.default_rng(5)
    for (b, h) in {(0, 0), (B - 1, H - 1), (B // 2, H // 2)}:
        rows = sample_rows(N, rng)
        q, k, v, _ = head_arrays(inp, b, h)
        kv = None if inp["seqlens"] is None else int(inp["seqlens"][b])
        ro, rl = head_forward_rows(q, k, v, w.scale, rows, w.causal, kv, inp["block_mask"],
                                   w.dropout_p, w.dropout_seed, b, h)
        go = f64(o[b, h])[rows]
        gl = lse[b, h].cpu().numpy().astype(np.float64)[rows]
        assert (np.abs(go - ro) <= 1e-2 + 2.0 ** -8 * np.abs(ro)).all()
        fin = np.isfinite(rl)
        assert np.array_equal(np.isfinite(gl), fin)
        assert np.abs(gl[fin] - rl[fin]).max() <= 1e-3


@pytest.mark.parametrize("name", NAMES)
def test_fullsize_dq_rows(lib, name):
    w, inp, o, lse, dq, dk, dv = run_workload(lib, name)
    B, H, N = w.B, w.H, w.N
    rng = np.random.default_rng(6)
    for (b, h) in {(0, 0), (B - 1, H - 1)}:
        rows = sample_rows(N, rng)
        q, k, v, do = head_arrays(inp, b, h)
        kv = None if inp["seqlens"] is None else int(inp["seqlens"][b])
        ref = head_backward_rows(q, k, v, do, w.scale, rows, w.causal, kv, inp["block_mask"],
                                 w.dropout_p, w.dropout_seed, b, h)
        assert rel_l2(f64(dq[b, h])[rows], ref) <= 2e-2


@pytest.mark.parametrize("name", NAMES)
def test_fullsize_dk_dv_columns(lib, name):
    w, inp, o, lse, dq, dk, dv = run_workload(lib, name)
    B, H, N = w.B, w.H, w.N
    rng = np.random.default_rng(7)
    b, h = B - 1, H - 1
    q, k, v, do = head_arrays(inp, b, h)
    kv = None if inp["seqlens"] is None else int(inp["seqlens"][b])
    bm = inp["block_mask"]
    rows = None
    if bm is not None:
        # key columns from two key blocks; only query blocks the mask keeps for
        # those key blocks can contribute (the others have P = 0 there)
        kb = [3, (N // 128) - 2]
        cols = np.concatenate([np.arange(c * 128, c * 128 + 128, 9) for c in kb])
        qblocks = np.nonzero(bm[:, kb].any(axis=1))[0]
        rows = np.concatenate([np.arange(r * 128, min(N, r * 128 + 128)) for r in qblocks])
    else:
        cols = sample_rows(N, rng)
    rdk, rdv = head_backward_cols(q, k, v, do, w.scale, cols, w.causal, kv, bm, w.dropout_p,
                                  w.dropout_seed, b, h, slab=512, rows=rows)
    assert rel_l2(f64(dk[b, h])[cols], rdk) <= 2e-2
    assert rel_l2(f64(dv[b, h])[cols], rdv) <= 2e-2


def test_fullsize_sparse_dk_sums_to_zero(lib):
    """sum_j dK_j = scale sum_i (sum_j dS_ij) Q_i = 0 for every head at 64K."""
    w, inp, o, lse, dq, dk, dv = run_workload(lib, "sparse")
    g = dk.float()
    s = g.sum(dim=2)                 # [B, H, d]
    tot = g.abs().sum(dim=2)         # [B, H, d]
    assert (s.abs() <= 1e-3 * tot + 1e-3).all()
    assert np.isfinite(f64(dq)).all() and np.isfinite(f64(dv)).all()
