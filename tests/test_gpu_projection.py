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
