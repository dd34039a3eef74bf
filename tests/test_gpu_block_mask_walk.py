"""The two ways the kernels walk a block mask: through the per-CTA bitmask
they gather in shared memory (the default) and byte by byte (the walk a mask
too long for the bitmask takes, forced here through the test-support switch).
Both visit the same tiles in the same order, so O, LSE, dK and dV must come
out bit for bit the same, and dQ equal up to the order of its fp32
reductions; the bitmask walk is also checked against the oracle by every
block-mask parity test."""

import numpy as np
import pytest

from io_aware_exact_20_b200.workloads import make_block_mask, make_qkvdo, make_seqlens

pytestmark = pytest.mark.gpu


def run_both(lib, q, k, v, do, **kw):
    import torch
    out = []
    for bitmap in (True, False):
        lib.set_block_mask_bitmap(bitmap)
        try:
            o, lse = lib.forward(q, k, v, **kw)
            dq, dk, dv = lib.backward(q, k, v, o, lse, do, **kw)
            torch.cuda.synchronize()
            assert lib.last_device_status() == 0
        finally:
            lib.set_block_mask_bitmap(True)
        out.append([x.float().cpu().numpy() for x in (o, lse, dq, dk, dv)])
    return out


@pytest.mark.parametrize("B,H,N,d,causal,lens,density,p", [
    (1, 2, 1000, 64, False, None, 0.3, 0.0),
    (2, 2, 777, 64, True, (100, 777), 0.5, 0.1),
    (1, 2, 900, 128, True, None, 0.4, 0.0),
    (2, 1, 1300, 128, False, (500, 1300), 0.25, 0.2),
])
def test_bitmask_walk_equals_byte_walk(lib, B, H, N, d, causal, lens, density, p):
    import torch
    q, k, v, do = (x.cuda() for x in make_qkvdo(B, H, N, d, 31))
    bm = make_block_mask(N, density, 32)
    bm[1, :] = 0  # a query tile that meets no key tile
    bm[:, 2] = 0  # a key tile that no query tile meets
    seqlens = None if lens is None else make_seqlens(B, lens[0], lens[1], 33)
    kw = dict(scale=d ** -0.5, causal=causal, seqlens=seqlens, dropout_p=p, seed=9,
              block_mask=torch.from_numpy(bm))
    (o1, l1, dq1, dk1, dv1), (o2, l2, dq2, dk2, dv2) = run_both(lib, q, k, v, do, **kw)
    for a, b in ((o1, o2), (l1, l2), (dk1, dk2), (dv1, dv2)):
        assert np.array_equal(a, b, equal_nan=True)
    scale = np.abs(dq1).max() + 1e-30
    assert np.abs(dq1 - dq2).max() <= 1e-2 * scale


def test_bitmask_walk_equals_byte_walk_packed(lib):
    """The same for a packed variable-length batch (the mask indexed by tile
    positions inside each sequence, N_q != N_k, causal, dropout, d = 64)."""
    import torch
    lq, lk = [300, 1, 700, 129], [500, 40, 650, 129]
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    g = torch.Generator().manual_seed(21)
    H, d = 2, 64
    q, do = (torch.randn(int(cu_q[-1]), H, d, generator=g).to(torch.bfloat16).cuda()
             for _ in range(2))
    k, v = (torch.randn(int(cu_k[-1]), H, d, generator=g).to(torch.bfloat16).cuda()
            for _ in range(2))
    bm = make_block_mask(700, 0.5, 22)[:, :6]
    bm[2, :] = 0
    kw = dict(layout="thd", cu_seqlens_q=cu_q, cu_seqlens_k=cu_k, max_seqlen_q=700,
              max_seqlen_k=650, causal=True, dropout_p=0.1, seed=5, block_mask=bm)
    out = []
    for bitmap in (True, False):
        lib.set_block_mask_bitmap(bitmap)
        try:
            o, lse = lib.forward_general(q, k, v, **kw)
            dq, dk, dv = lib.backward_general(q, k, v, o, lse, do, **kw)
            torch.cuda.synchronize()
            assert lib.last_device_status() == 0
        finally:
            lib.set_block_mask_bitmap(True)
        out.append([x.float().cpu().numpy() for x in (o, lse, dq, dk, dv)])
    (o1, l1, dq1, dk1, dv1), (o2, l2, dq2, dk2, dv2) = out
    for a, b in ((o1, o2), (l1, l2), (dk1, dk2), (dv1, dv2)):
        assert np.array_equal(a, b, equal_nan=True)
    assert np.abs(dq1 - dq2).max() <= 1e-2 * (np.abs(dq1).max() + 1e-30)
