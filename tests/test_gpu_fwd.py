"""Forward parity: the CUDA kernels (through the C ABI) against the float64 oracle.

Tolerances: O max-abs <= 1e-2 and LSE max-abs <= 1e-3 (bf16 inputs, fp32
accumulation, P rounded to bf16 before the P V product).  O is stored as
bf16, whose round-to-nearest adds up to 2^-8 |O| on top of the computed
value's error (half a bf16 ulp, 0.0156 once |O| >= 4, which dropout's
1 / (keep probability) and rows with few keys reach), so the O bound is
1e-2 + 2^-8 |O_ref|.  Rows without a valid key must give O = 0 and
LSE = -inf exactly; dropout keep bits are bit-exact.
"""

import numpy as np
import pytest

from oracle import attention_forward, dropout_keep, dropout_scale
from io_aware_exact_20_b200.workloads import make_block_mask, make_qkvdo, make_seqlens

pytestmark = pytest.mark.gpu

O_TOL = 1e-2
LSE_TOL = 1e-3


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def run_case(fa, B, H, N, d, causal=False, lens=None, density=None, p=0.0, seed=11,
             data_seed=1, scale=None):
    import torch
    q, k, v, _ = make_qkvdo(B, H, N, d, data_seed)
    seqlens = None if lens is None else make_seqlens(B, lens[0], lens[1], data_seed + 1)
    bm = None if density is None else make_block_mask(N, density, data_seed + 2)
    scale = d ** -0.5 if scale is None else scale
    dq, dk, dv = (x.cuda() for x in (q, k, v))
    o, lse = fa.forward(dq, dk, dv, scale=scale, causal=causal, seqlens=seqlens,
                        dropout_p=p, seed=seed, block_mask=bm)
    torch.cuda.synchronize()
    assert fa.last_device_status() == 0
    ro, rl = attention_forward(f64(q), f64(k), f64(v), scale, causal, seqlens, p, seed, bm)
    return f64(o), lse.cpu().numpy().astype(np.float64), ro, rl


def compare(o, lse, ro, rl, record=None):
    """Checks O and LSE against the oracle.  The strict bound on O
    (max-abs 1e-2) is asserted wherever bf16 storage can meet it (|O_ref| < 2,
    half an ulp <= 2^-8 |O| < 0.0079); everywhere the bound is
    1e-2 + 2^-8 |O_ref|.  The strict max-abs error over all elements is
    returned (and recorded) so the slack actually used is visible."""
    assert np.isfinite(o).all()
    empty = np.isneginf(rl)
    assert np.array_equal(np.isneginf(lse), empty), "rows without keys must have LSE = -inf"
    assert (o[empty] == 0).all()
    diff = np.abs(o - ro)
    err_o = diff.max()
    small = np.abs(ro) < 2.0
    err_small = diff[small].max() if small.any() else 0.0
    excess = (diff - (O_TOL + 2.0 ** -8 * np.abs(ro))).max()
    err_l = np.abs(lse[~empty] - rl[~empty]).max() if (~empty).any() else 0.0
    if record is not None:
        record(o_max_abs=float(err_o), o_max_abs_where_abs_ref_lt_2=float(err_small),
               o_max_abs_ref=float(np.abs(ro).max()), lse_max_abs=float(err_l))
    assert err_small <= O_TOL, ("strict O bound", err_small)
    assert excess <= 0, (err_o, excess)
    assert err_l <= LSE_TOL, err_l
    return err_o, err_l


CASES = [
    # B, H, N, d, causal, key lengths, block density, dropout p
    (1, 2, 128, 64, False, None, None, 0.0),       # the tiny exact workload
    (1, 1, 1, 64, False, None, None, 0.0),         # a single row and key
    (1, 1, 129, 128, True, None, None, 0.0),       # one row into the second tile
    (2, 3, 300, 64, True, None, None, 0.0),        # ragged tail, causal
    (2, 2, 384, 128, False, None, None, 0.0),
    (2, 2, 520, 128, True, None, None, 0.0),
    (3, 2, 400, 64, False, (1, 400), None, 0.0),   # key padding incl. very short keys
    (2, 2, 333, 64, True, (0, 60), None, 0.0),     # lengths down to 0: empty rows
    (1, 2, 1024, 64, False, None, 0.25, 0.0),      # block sparse
    (1, 2, 640, 128, True, (300, 640), 0.5, 0.0),  # every mask at once
    (2, 2, 256, 64, True, None, None, 0.1),        # dropout
    (2, 2, 384, 128, False, (100, 384), None, 0.2),
    (1, 3, 700, 64, True, (500, 700), 0.4, 0.3),
    # d = 64 rows longer than 4096 (many K/V tiles per key-split stream)
    (1, 1, 4200, 64, False, None, 0.3, 0.0),
    (1, 2, 4224, 64, True, None, None, 0.1),
    (1, 1, 4400, 64, True, (2000, 4400), 0.4, 0.0),
]


@pytest.mark.parametrize("B,H,N,d,causal,lens,density,p", CASES)
def test_forward_matches_oracle(lib, parity_record, B, H, N, d, causal, lens, density, p):
    o, lse, ro, rl = run_case(lib, B, H, N, d, causal, lens, density, p)
    compare(o, lse, ro, rl, parity_record)


def block_mask_with_holes(N, seed):
    """A block mask whose diagonal is not all set: query tile 1 keeps no key
    block (its rows have no valid key), key tile 2 is kept by no query tile,
    and the diagonal blocks (0, 0) and (3, 3) are removed.  Legal input; the
    workload generator never makes it (it always keeps the diagonal)."""
    bm = make_block_mask(N, 0.5, seed)
    bm[1, :] = 0
    bm[:, 2] = 0
    bm[0, 0] = 0
    bm[3, 3] = 0
    bm[4, 4] = 1
    return bm


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("p", [0.0, 0.1])
def test_forward_block_mask_without_diagonal(lib, parity_record, d, causal, p):
    import torch
    B, H, N = 2, 2, 600
    q, k, v, _ = make_qkvdo(B, H, N, d, 31)
    bm = block_mask_with_holes(N, 32)
    scale = d ** -0.5
    o, lse = lib.forward(q.cuda(), k.cuda(), v.cuda(), scale=scale, causal=causal, dropout_p=p,
                         seed=5, block_mask=bm)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    ro, rl = attention_forward(f64(q), f64(k), f64(v), scale, causal, None, p, 5, bm)
    o, lse = f64(o), lse.cpu().numpy().astype(np.float64)
    assert np.isneginf(rl[:, :, 128:256]).all()  # query tile 1 is empty
    compare(o, lse, ro, rl, parity_record)
    assert (o[:, :, 128:256] == 0).all()


def test_forward_long_rows_many_tiles(lib):
    """Many K/V tiles per row so the lazily moved maximum is exercised: keys
    with a growing bias make the row maximum increase tile after tile."""
    import torch
    B, H, N, d = 1, 2, 2048, 64
    q, k, v, _ = make_qkvdo(B, H, N, d, 5)
    ramp = torch.linspace(0, 6, N).to(torch.bfloat16)
    q = q.clone()
    q[..., 0] = 4.0
    k = k.clone()
    k[..., 0] = ramp  # score grows with j: a new maximum in every tile
    o, lse = lib.forward(q.cuda(), k.cuda(), v.cuda(), causal=False)
    ro, rl = attention_forward(f64(q), f64(k), f64(v), d ** -0.5)
    compare(f64(o), lse.cpu().numpy().astype(np.float64), ro, rl)


@pytest.mark.parametrize("c", [20480.0, -20480.0])
def test_forward_safe_softmax_at_plus_minus_20000(lib, c):
    """Scores of about +-20000 on every key (the pages' overflow / underflow
    example): the result is the mean of V, with no inf or nan."""
    import torch
    B, H, N, d = 1, 1, 256, 64
    _, _, v, _ = make_qkvdo(B, H, N, d, 6)
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16)
    q[..., 0] = c
    k = torch.zeros(B, H, N, d, dtype=torch.bfloat16)
    k[..., 0] = 1.0
    o, lse = lib.forward(q.cuda(), k.cuda(), v.cuda(), scale=1.0)
    o, lse = f64(o), lse.cpu().numpy().astype(np.float64)
    ro, rl = attention_forward(f64(q), f64(k), f64(v), 1.0)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    assert (np.abs(o - ro) <= O_TOL + 2.0 ** -8 * np.abs(ro)).all()
    # LSE ~ c + ln N: fp32 resolution at 2e4 is ~2e-3, so compare relatively
    assert np.abs(lse - rl).max() <= 4e-3


def test_dropout_mask_bits_match_oracle(lib):
    B, H, N = 2, 3, 257
    for p, seed in ((0.1, 0x5EED0002), (0.5, 123456789012345)):
        keep = lib.dropout_mask(B, H, N, p, seed).cpu().numpy().astype(bool)
        for b in range(B):
            for h in range(H):
                want = dropout_keep(seed, p, b, h, np.arange(N), N)
                assert np.array_equal(keep[b, h], want)


@pytest.mark.parametrize("d", [64, 128])
def test_forward_kernel_dropout_bits_exact(lib, d):
    """Q = 0 makes P uniform (1/N); V rows one-hot over a window of d keys then
    give O[i, c] = keep(i, j0 + c) / (N q), q the keep probability: every keep bit the real
    forward kernel used is read back and compared with the oracle's."""
    import torch
    B, H, N, p, seed = 1, 2, 256, 0.1, 0x5EED0002
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    k = torch.randn(B, H, N, d, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16).cuda()
    level = dropout_scale(p) / N
    for j0 in range(0, N, d):
        v = torch.zeros(B, H, N, d, dtype=torch.bfloat16)
        for c in range(d):
            v[:, :, j0 + c, c] = 1.0
        o, _ = lib.forward(q, k, v.cuda(), dropout_p=p, seed=seed)
        got = f64(o) > 0.5 * level
        for b in range(B):
            for h in range(H):
                want = dropout_keep(seed, p, b, h, np.arange(N), N)[:, j0:j0 + d]
                assert np.array_equal(got[b, h], want)
        nz = f64(o)[got]
        assert np.abs(nz - level).max() < 0.01 * level
