"""The unfused standard-attention baseline that bench.py times beside the
fused kernels computes the same thing: its O and gradients match the float64
oracle (no dropout: the baseline draws dropout bits from torch's generator).
bf16 tensors and bf16 S / P in device memory, so the bounds are those of the
fused path's parity tests, loosened for O by the bf16 rounding of P and O."""

import numpy as np
import pytest

from oracle import attention_backward, attention_forward
from io_aware_exact_20_b200.workloads import make_block_mask, make_qkvdo, make_seqlens

pytestmark = pytest.mark.gpu


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("causal,lens,density", [(True, None, None), (False, (200, 384), None),
                                                 (False, None, 0.4)])
def test_unfused_baseline_matches_oracle(causal, lens, density):
    import torch
    from baselines.unfused_attention import UnfusedStep
    B, H, N, d = 2, 2, 384, 64
    q, k, v, do = make_qkvdo(B, H, N, d, 41)
    sl = None if lens is None else make_seqlens(B, lens[0], lens[1], 42)
    bm = None if density is None else make_block_mask(N, density, 43)
    scale = d ** -0.5
    step = UnfusedStep(q.cuda(), k.cuda(), v.cuda(), do.cuda(), scale, causal, sl, 0.0, bm)
    o, dq, dk, dv = step()
    torch.cuda.synchronize()
    ro, _ = attention_forward(f64(q), f64(k), f64(v), scale, causal, sl, 0.0, 0, bm)
    rg = attention_backward(f64(q), f64(k), f64(v), f64(do), scale, causal, sl, 0.0, 0, bm)
    assert np.abs(f64(o) - ro).max() <= 2e-2
    for a, r in zip((dq, dk, dv), rg):
        assert np.linalg.norm(f64(a) - r) / np.linalg.norm(r) <= 2e-2
