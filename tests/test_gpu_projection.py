"""Fused QKV projection (fa_qkv_projection) against the float64 oracle:
Y = X W^T + bias split into head-major Q, K, V.  bf16 inputs, fp32
accumulation, one rounding to bf16: |error| <= 2^-8 |Y_ref| + 1e-3."""

import numpy as np
import pytest

from oracle import qkv_projection

pytestmark = pytest.mark.gpu


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("B,N,H,d,dm,bias", [
    (2, 300, 4, 64, 200, True),     # ragged token tile, model dim not a multiple of 64
    (1, 128, 2, 64, 64, False),     # one tile, one K chunk
    (3, 257, 3, 128, 768, True),
    (8, 1024, 12, 64, 768, True),   # GPT-2-small shape
])
def test_qkv_projection_matches_oracle(lib, B, N, H, d, dm, bias):
    import torch
    g = torch.Generator().manual_seed(B * 1000 + dm)
    x = torch.randn(B * N, dm, generator=g).to(torch.bfloat16)
    w = (torch.randn(3 * H * d, dm, generator=g) / dm ** 0.5).to(torch.bfloat16)
    b = torch.randn(3 * H * d, generator=g).to(torch.bfloat16) if bias else None
    q, k, v = lib.qkv_projection(x.cuda(), w.cuda(), None if b is None else b.cuda(), B, H, d)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    ref = qkv_projection(f64(x), f64(w), None if b is None else f64(b), B, H, d)
    for got, r in zip((q, k, v), ref):
        err = np.abs(f64(got) - r)
        assert (err <= 2.0 ** -8 * np.abs(r) + 1e-3).all(), err.max()


def test_projection_output_feeds_attention_back_to_back(lib):
    """The projection and the attention forward / backward launched back to
    back on one stream (each may start launching under its predecessor's last
    wave, and must wait for it before reading): the attention reads the Q, K,
    V the projection has just written, and a torch kernel that rewrites V in
    between is seen by the next call."""
    import torch
    from oracle import attention_forward
    B, N, H, d, dm = 2, 384, 2, 64, 256
    g = torch.Generator().manual_seed(77)
    x = torch.randn(B * N, dm, generator=g).to(torch.bfloat16).cuda()
    w = (torch.randn(3 * H * d, dm, generator=g) / dm ** 0.5).to(torch.bfloat16).cuda()
    q, k, v = lib.qkv_projection(x, w, None, B, H, d)
    o1, _ = lib.forward(q, k, v, causal=True)
    v.mul_(-2.0)                      # a torch kernel between two library calls
    o2, lse2 = lib.forward(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    rq, rk, rv = qkv_projection(f64(x), f64(w), None, B, H, d)
    # the oracle on the bf16 values the kernels actually read
    qb, kb, vb = (f64(t) for t in (q, k, v))
    ro1, _ = attention_forward(qb, kb, -0.5 * vb, d ** -0.5, True)
    ro2, rl2 = attention_forward(qb, kb, vb, d ** -0.5, True)
    assert np.abs(f64(o1) - ro1).max() <= 1e-2 + 2.0 ** -8 * np.abs(ro1).max()
    assert np.abs(f64(o2) - ro2).max() <= 1e-2 + 2.0 ** -8 * np.abs(ro2).max()
    assert np.abs(lse2.cpu().numpy() - rl2).max() <= 1e-3
    for got, r in zip((q, k), (rq, rk)):
        assert (np.abs(f64(got) - r) <= 2.0 ** -8 * np.abs(r) + 1e-3).all()
