"""The 256-wide forward (head dims 192 and 256, forward only) against the
float64 oracle: the classic layout, strided and packed layouts, every mask,
dropout, rows long enough that the single K/V stage is refilled many times
(K and V released separately), and the backward's refusal of these dims."""

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


def test_wide_backward_is_refused(lib):
    """The backward entry points refuse d = 256 (no launch, FA_ERR_UNSUPPORTED)."""
    import torch
    q, k, v, do = (x.cuda() for x in make_qkvdo(1, 1, 128, 256, 3))
    o, lse = lib.forward(q, k, v)
    torch.cuda.synchronize()
    with pytest.raises(lib.FaError):
        lib.backward(q, k, v, o, lse, do)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0


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
