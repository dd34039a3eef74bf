"""Host-side logic of bench.py that needs no GPU: the effective FLOP share of
masked workloads and the roofline fraction taken on the effective count (so a
block-sparse run cannot report more than the tensor peak)."""

import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_effective_fraction_of_the_workloads():
    import bench
    from io_aware_exact_20_b200.workloads import WORKLOADS, make_block_mask, make_seqlens
    w = WORKLOADS["bert"]
    lens = make_seqlens(w.B, *w.seqlen_range, w.len_seed)
    assert bench.effective_fraction({"seqlens": lens}, w) == pytest.approx(lens.mean() / w.N)
    w = WORKLOADS["sparse"]
    bm = make_block_mask(w.N, w.block_density, w.mask_seed)
    f = bench.effective_fraction({"block_mask": bm}, w)
    assert f == pytest.approx(bm.mean())
    assert 0.12 < f < 0.135  # 1/8 plus the diagonal
    assert bench.effective_fraction({}, WORKLOADS["long128"]) == 1.0


def test_roofline_fraction_uses_the_effective_count():
    import bench
    from io_aware_exact_20_b200.workloads import WORKLOADS, attention_flops
    w = WORKLOADS["sparse"]
    f_fwd, f_bwd = attention_flops(w.B, w.H, w.N, w.d, w.causal)
    eff = 0.127
    # timings of the size the nominal count would turn into 2.7x the peak
    main_ms = f_bwd / (2.7 * 1590e12) * 1e3
    s = bench.kernel_summary(w, eff, 0.5 * main_ms, 0.01, main_ms, 0.01, 1590.0)
    assert s["dominant"]["kernel"] == "bwd_main_kernel"
    assert s["dominant"]["frac"] == pytest.approx(2.7 * eff)
    assert s["dominant"]["frac"] < 1.0
    assert s["nominal_tflops"]["bwd_main"] == pytest.approx(2.7 * 1590.0)


def test_job_throughput_and_reference_sample_accounting():
    import bench
    from io_aware_exact_20_b200.workloads import WORKLOADS, attention_flops
    assert bench.job_throughput(2, 1e12, 5, 1000.0) == pytest.approx(10.0)
    # one 256-row slab stands for its share of the nominal count
    w = WORKLOADS["long128"]
    ff, fb = attention_flops(1, 1, w.N, w.d, w.causal)
    assert (ff + fb) * bench.SLAB / w.N == pytest.approx((ff + fb) / 64)
