"""The 256-wide kernels (head dims 192 and 256) against the float64 oracle:
the forward in the classic layout, strided and packed layouts, every mask,
dropout, rows long enough that the single K/V stage is refilled many times
(K and V released separately); the backward (two CTAs per key tile, each
owning half of dK / dV / dQ's columns, Q and dO through a ring of 64-column
panels) in the same layouts and over enough query tiles to cycle the ring
many times.  Bounds as in the other parity tests."""

import numpy as np
import pytest

from oracle import attention_forward
from io_aware_exact_20_b200.workloads import make_qkvdo
from oracle.varlen_ref import attention_forward_varlen
from test_gpu_fwd import compare, f64, run_case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,N,d,causal,lens,density,p", [
    (1, 2, 128, 256, False, None, None, 0.0),
    (2, 2, 300, 256, True, None, None, 0.1),        # ragged tail, dropout
    (1, 2, 4096, 256, True, None, None, 0.0),       # 32 K/V tiles through one stage
    (2, 1, 1000, 256, False, (100, 1000), 0.4, 0.2),  # every mask
    (1, 3, 777, 192, True, (300, 777), None, 0.1),  # d = 192 on zero columns
])
def test_wide_forward_matches_oracle(lib, parity_record, B, H, N, d, causal, lens, density, p):
    o, lse, ro, rl = run_case(lib, B, H, N, d, causal, lens, density, p)
    compare(o, lse, ro, rl, parity_record)


def test_wide_forward_block_mask_with_empty_rows(lib, parity_record):
    """A query tile the block mask leaves without keys gets O = 0, LSE = -inf."""
    import torch
    B, H, N, d = 1, 2, 640, 256
    q, k, v, _ = make_qkvdo(B, H, N, d, 5)
    bm = np.ones((5, 5), dtype=np.uint8)
    bm[2, :] = 0
    bm[:, 3] = 0
    o, lse = lib.forward(q.cuda(), k.cuda(), v.cuda(), causal=True, dropout_p=0.1, seed=4,
                         block_mask=bm)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    ro, rl = attention_forward(f64(q), f64(k), f64(v), d ** -0.5, True, None, 0.1, 4, bm)
    compare(f64(o), lse.cpu().numpy().astype(np.float64), ro, rl, parity_record)
    assert np.all(np.isneginf(lse.cpu().numpy()[:, :, 256:384]))


def test_wide_forward_general_layouts(lib, parity_record):
    """Token-major strides with N_q != N_k (bottom-right causal), and a packed
    variable-length batch, at d = 256."""
    import torch
    B, H, Nq, Nk, d = 2, 2, 200, 520, 256
    qh = make_qkvdo(B, H, Nq, d, 6)[0]
    _, kh, vh, _ = make_qkvdo(B, H, Nk, d, 7)
    t = lambda x: x.transpose(1, 2).contiguous().cuda()  # noqa: E731  [B, N, H, d]
    o, lse = lib.forward_general(t(qh), t(kh), t(vh), layout="bshd", causal=True,
                                 dropout_p=0.1, seed=8)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    ro, rl = attention_forward(f64(qh), f64(kh), f64(vh), d ** -0.5, True, None, 0.1, 8)
    compare(f64(o.transpose(1, 2)), lse.cpu().numpy().astype(np.float64), ro, rl, parity_record)

    lq, lk = [129, 0, 300], [200, 5, 300]
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    g = torch.Generator().manual_seed(9)
    pq = torch.randn(int(cu_q[-1]), H, d, generator=g).to(torch.bfloat16)
    pk, pv = (torch.randn(int(cu_k[-1]), H, d, generator=g).to(torch.bfloat16) for _ in range(2))
    o, lse = lib.forward_general(pq.cuda(), pk.cuda(), pv.cuda(), layout="thd", cu_seqlens_q=cu_q,
                                 cu_seqlens_k=cu_k, max_seqlen_q=300, max_seqlen_k=300,
                                 causal=True, dropout_p=0.1, seed=10)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    ro, rl = attention_forward_varlen(f64(pq), f64(pk), f64(pv), cu_q, cu_k, d ** -0.5, True,
                                      None, 0.1, 10)
    # packed O [T, H, d] and LSE [H, T] viewed as one batch entry [1, H, T, d] / [1, H, T]
    as_bhsd = lambda x: np.transpose(x, (1, 0, 2))[None]  # noqa: E731
    compare(as_bhsd(f64(o)), lse.cpu().numpy().astype(np.float64)[None], as_bhsd(ro), rl[None],
            parity_record)


def _rel_l2(a, r):
    n = np.linalg.norm(r)
    return np.linalg.norm(a - r) / n if n > 0 else np.linalg.norm(a)


def _check_grads(got, ref, record):
    errs = {}
    for name, a, r in zip(("dq", "dk", "dv"), got, ref):
        assert np.isfinite(a).all(), name
        errs[name] = _rel_l2(a, r)
    record(**{f"{k}_rel_l2": float(v) for k, v in errs.items()})
    for name, e in errs.items():
        assert e <= 2e-2, (name, e)


@pytest.mark.parametrize("N,d,causal,p", [
    (4096, 256, True, 0.0),    # 32 query tiles for the first key tile: the ring turns 96 times
    (2176, 192, False, 0.1),   # 17 x 128 rows, dropout (the one-pass P / dS order)
])
def test_wide_backward_long_rows(lib, parity_record, N, d, causal, p):
    import torch
    from oracle import attention_backward
    q, k, v, do = make_qkvdo(1, 2, N, d, 14)
    kw = dict(causal=causal, dropout_p=p, seed=15)
    gq, gk, gv, gdo = (x.cuda() for x in (q, k, v, do))
    o, lse = lib.forward(gq, gk, gv, **kw)
    grads = lib.backward(gq, gk, gv, o, lse, gdo, **kw)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    ref = attention_backward(f64(q), f64(k), f64(v), f64(do), d ** -0.5, causal, None, p, 15)
    _check_grads(tuple(f64(x) for x in grads), ref, parity_record)


def test_wide_backward_general_layouts(lib, parity_record):
    """Token-major strides with N_q != N_k (bottom-right causal) and a packed
    variable-length batch with an empty sequence, at d = 256."""
    import torch
    from oracle import attention_backward
    from oracle.varlen_ref import attention_backward_varlen
    B, H, Nq, Nk, d = 2, 2, 200, 520, 256
    qh, doh = make_qkvdo(B, H, Nq, d, 16)[0], make_qkvdo(B, H, Nq, d, 17)[3]
    _, kh, vh, _ = make_qkvdo(B, H, Nk, d, 18)
    t = lambda x: x.transpose(1, 2).contiguous().cuda()  # noqa: E731  [B, N, H, d]
    kw = dict(layout="bshd", causal=True, dropout_p=0.1, seed=19)
    q, k, v, do = t(qh), t(kh), t(vh), t(doh)
    o, lse = lib.forward_general(q, k, v, **kw)
    grads = lib.backward_general(q, k, v, o, lse, do, **kw)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    ref = attention_backward(f64(qh), f64(kh), f64(vh), f64(doh), d ** -0.5, True, None, 0.1, 19)
    _check_grads(tuple(f64(x.transpose(1, 2)) for x in grads), ref, parity_record)

    lq, lk = [129, 0, 300], [200, 5, 300]
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    g = torch.Generator().manual_seed(20)
    pq, pdo = (torch.randn(int(cu_q[-1]), H, d, generator=g).to(torch.bfloat16) for _ in range(2))
    pk, pv = (torch.randn(int(cu_k[-1]), H, d, generator=g).to(torch.bfloat16) for _ in range(2))
    kw = dict(layout="thd", cu_seqlens_q=cu_q, cu_seqlens_k=cu_k, max_seqlen_q=300,
              max_seqlen_k=300, causal=True, dropout_p=0.1, seed=21)
    q, k, v, do = (x.cuda() for x in (pq, pk, pv, pdo))
    o, lse = lib.forward_general(q, k, v, **kw)
    grads = lib.backward_general(q, k, v, o, lse, do, **kw)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    ref = attention_backward_varlen(f64(pq), f64(pk), f64(pv), f64(pdo), cu_q, cu_k, d ** -0.5,
                                    True, None, 0.1, 21)
    _check_grads(tuple(f64(x) for x in grads), ref, parity_record)


def test_wide_forward_bitmask_walk_equals_byte_walk(lib):
    """The 256-wide forward walks a block mask through its shared-memory
    bitmask or byte by byte (test-support switch) with identical O and LSE."""
    import torch
    from io_aware_exact_20_b200.workloads import make_block_mask
    q, k, v, _ = (x.cuda() for x in make_qkvdo(1, 2, 1100, 256, 12))
    bm = make_block_mask(1100, 0.4, 13)
    bm[4, :] = 0
    out = []
    for bitmap in (True, False):
        lib.set_block_mask_bitmap(bitmap)
        try:
            o, lse = lib.forward(q, k, v, causal=True, dropout_p=0.1, seed=2, block_mask=bm)
            torch.cuda.synchronize()
            assert lib.last_device_status() == 0
        finally:
            lib.set_block_mask_bitmap(True)
        out.append((o.float().cpu().numpy(), lse.cpu().numpy()))
    assert np.array_equal(out[0][0], out[1][0])
    assert np.array_equal(out[0][1], out[1][1])
