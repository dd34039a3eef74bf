"""Grouped K / V heads (k, v with H_kv heads, query head h reading K / V head
h // (H / H_kv)) through fa_fwd_ex / fa_bwd_ex against the float64 oracle:
the classic, token-major and packed layouts, the 64-, 128- and 256-wide
kernels, causal and key-padding masks, a block mask and dropout.  The backward
walks the query heads of a group inside one thread block, so dK and dV of a
shared head accumulate over the group without atomics.  Bounds as in the
other parity tests."""

import numpy as np
import pytest

from oracle import (
    attention_backward_gqa,
    attention_backward_varlen,
    attention_forward_gqa,
    attention_forward_varlen,
    gqa_expand,
    gqa_reduce,
)
from test_gpu_fwd import compare
from test_gpu_general import check_grads, f64, randn

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("layout", ["bhsd", "bshd"])
@pytest.mark.parametrize("B,H,Hkv,Nq,Nk,d,causal,lens,density,p", [
    (2, 4, 2, 300, 300, 64, True, None, None, 0.1),
    (1, 4, 1, 260, 260, 128, False, (100, 260), None, 0.0),     # one K / V head (G = 4)
    (1, 6, 3, 200, 520, 96, True, None, None, 0.2),             # N_q != N_k
    (2, 4, 2, 384, 384, 64, False, None, 0.5, 0.1),             # block mask
    (1, 4, 2, 300, 300, 256, True, None, None, 0.1),            # the 256-wide kernels
    (1, 2, 1, 129, 129, 192, False, None, None, 0.0),
])
def test_gqa_matches_oracle(lib, parity_record, layout, B, H, Hkv, Nq, Nk, d, causal, lens,
                            density, p):
    import torch
    from io_aware_exact_20_b200.workloads import make_seqlens
    qh, doh = randn((B, H, Nq, d), 41), randn((B, H, Nq, d), 42)
    kh, vh = randn((B, Hkv, Nk, d), 43), randn((B, Hkv, Nk, d), 44)
    seqlens = None if lens is None else make_seqlens(B, lens[0], lens[1], 45)
    bm = None
    if density is not None:
        nbq, nbk = (Nq + 127) // 128, (Nk + 127) // 128
        bm = (np.random.default_rng(46).random((nbq, nbk)) < density).astype(np.uint8)
        bm[0, :] = 1
        bm[:, -1] = 0  # a key tile no query tile meets: dK = dV = 0 there
    scale, seed = d ** -0.5, 0x5EED00A1
    kw = dict(layout=layout, scale=scale, causal=causal, seqlens_k=seqlens, dropout_p=p,
              seed=seed, block_mask=bm)

    def dev(x):
        x = x.cuda()
        return x.transpose(1, 2).contiguous() if layout == "bshd" else x

    def host(x):
        return f64(x.transpose(1, 2) if layout == "bshd" else x)

    q, k, v, do = dev(qh), dev(kh), dev(vh), dev(doh)
    o, lse = lib.forward_general(q, k, v, **kw)
    dq, dk, dv = lib.backward_general(q, k, v, o, lse, do, **kw)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    assert tuple(dk.shape) == tuple(k.shape) and tuple(dv.shape) == tuple(v.shape)
    args = (scale, causal, seqlens, p, seed, bm)
    ro, rl = attention_forward_gqa(f64(qh), f64(kh), f64(vh), *args)
    compare(host(o), f64(lse), ro, rl, parity_record)
    rg = attention_backward_gqa(f64(qh), f64(kh), f64(vh), f64(doh), *args)
    check_grads((host(dq), host(dk), host(dv)), rg, parity_record)


def test_gqa_packed_batch(lib, parity_record):
    """Packed sequences (one empty) with one K / V head for four query heads."""
    import torch
    H, Hkv, d = 4, 1, 64
    lq, lk = [129, 0, 300], [200, 5, 300]
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    g = torch.Generator().manual_seed(47)
    pq, pdo = (torch.randn(int(cu_q[-1]), H, d, generator=g).to(torch.bfloat16) for _ in range(2))
    pk, pv = (torch.randn(int(cu_k[-1]), Hkv, d, generator=g).to(torch.bfloat16) for _ in range(2))
    kw = dict(layout="thd", cu_seqlens_q=cu_q, cu_seqlens_k=cu_k, max_seqlen_q=300,
              max_seqlen_k=300, causal=True, dropout_p=0.1, seed=48)
    q, k, v, do = (x.cuda() for x in (pq, pk, pv, pdo))
    o, lse = lib.forward_general(q, k, v, **kw)
    grads = lib.backward_general(q, k, v, o, lse, do, **kw)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    G = H // Hkv
    ek, ev = gqa_expand(f64(pk), G), gqa_expand(f64(pv), G)  # packed [T, H, d]: heads on axis 1
    ro, rl = attention_forward_varlen(f64(pq), ek, ev, cu_q, cu_k, d ** -0.5, True, None, 0.1, 48)
    as_bhsd = lambda x: np.transpose(x, (1, 0, 2))[None]  # noqa: E731
    compare(as_bhsd(f64(o)), f64(lse)[None], as_bhsd(ro), rl[None], parity_record)
    rq, rk, rv = attention_backward_varlen(f64(pq), ek, ev, f64(pdo), cu_q, cu_k, d ** -0.5, True,
                                           None, 0.1, 48)
    check_grads(tuple(f64(x) for x in grads), (rq, gqa_reduce(rk, G), gqa_reduce(rv, G)),
                parity_record)


def test_gqa_forward_equals_repeated_heads(lib):
    """The grouped forward reads the same numbers as a call with each K / V
    head repeated for its query heads: O and LSE are identical bit for bit."""
    import torch
    B, H, Hkv, N, d = 2, 6, 2, 333, 128
    q = randn((B, H, N, d), 49).cuda()
    k, v = randn((B, Hkv, N, d), 50).cuda(), randn((B, Hkv, N, d), 51).cuda()
    kw = dict(causal=True, dropout_p=0.1, seed=52)
    o1, l1 = lib.forward_general(q, k, v, **kw)
    rep = lambda x: x.repeat_interleave(H // Hkv, dim=1).contiguous()  # noqa: E731
    o2, l2 = lib.forward_general(q, rep(k), rep(v), **kw)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("parts", [1, 2, 4])
@pytest.mark.parametrize("d", [64, 128])
def test_gqa_backward_split_parts(lib, parity_record, parts, d):
    """A unit of the grouped backward walks its group's query heads in one
    thread block (parts = 1: dK / dV accumulate in TMEM and are stored once),
    or is split into parts that each walk their share and add dK / dV into fp32
    accumulators converted at the end; every split gives the oracle's result."""
    import torch
    B, H, Hkv, N = 1, 8, 2, 520
    qh, doh = randn((B, H, N, d), 61), randn((B, H, N, d), 62)
    kh, vh = randn((B, Hkv, N, d), 63), randn((B, Hkv, N, d), 64)
    kw = dict(causal=True, dropout_p=0.1, seed=65)
    q, k, v, do = (x.cuda() for x in (qh, kh, vh, doh))
    lib.set_gqa_split(parts)
    try:
        o, lse = lib.forward_general(q, k, v, **kw)
        grads = lib.backward_general(q, k, v, o, lse, do, **kw)
        torch.cuda.synchronize()
        assert lib.last_device_status() == 0
    finally:
        lib.set_gqa_split(0)
    args = (d ** -0.5, True, None, 0.1, 65)
    rg = attention_backward_gqa(f64(qh), f64(kh), f64(vh), f64(doh), *args)
    check_grads(tuple(f64(x) for x in grads), rg, parity_record)


def test_gqa_split_backward_is_repeatable(lib):
    """Split units write their partial dK / dV to slices summed in a fixed
    order: two runs give the same dK and dV bits."""
    import torch
    B, H, Hkv, N, d = 1, 8, 2, 640, 128
    q, do = randn((B, H, N, d), 71).cuda(), randn((B, H, N, d), 72).cuda()
    k, v = randn((B, Hkv, N, d), 73).cuda(), randn((B, Hkv, N, d), 74).cuda()
    kw = dict(causal=True, dropout_p=0.1, seed=75)
    lib.set_gqa_split(4)
    try:
        o, lse = lib.forward_general(q, k, v, **kw)
        a = lib.backward_general(q, k, v, o, lse, do, **kw)
        b = lib.backward_general(q, k, v, o, lse, do, **kw)
        torch.cuda.synchronize()
        assert lib.last_device_status() == 0
    finally:
        lib.set_gqa_split(0)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
