"""The partial-result kernels (fa_merge_partial, fa_accumulate_bf16,
fa_convert_f32_bf16) against the oracle's merge and against exact fp32 / bf16
arithmetic, for every head dim and ragged row counts."""

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _lse(rng, rows, empty_frac):
    lse = rng.normal(0.0, 3.0, rows).astype(np.float32)
    lse[rng.random(rows) < empty_frac] = -np.inf
    return lse


@pytest.mark.parametrize("d", [32, 64, 96, 128, 192, 256])
@pytest.mark.parametrize("rows", [1, 31, 777])
def test_merge_partial_matches_the_oracle(lib, d, rows):
    """Each row of O_acc / LSE_acc merged with its part, empty parts (LSE = -inf)
    on either side or both, against the oracle's merge in float64."""
    import torch

    from oracle import merge_partials
    rng = np.random.default_rng(1000 * d + rows)
    o_acc = rng.normal(size=(rows, d)).astype(np.float32)
    o_part = torch.from_numpy(rng.normal(size=(rows, d)).astype(np.float32)).bfloat16()
    lse_acc, lse_part = _lse(rng, rows, 0.2), _lse(rng, rows, 0.2)
    ro, rl = merge_partials(o_acc, lse_acc, o_part.float().numpy(), lse_part)
    # an empty accumulator's O is not read: the oracle's weight on it is 0 too
    a = torch.from_numpy(o_acc).cuda()
    la = torch.from_numpy(lse_acc).cuda()
    lib.merge_partial(a, la, o_part.cuda(), torch.from_numpy(lse_part).cuda())
    torch.cuda.synchronize()
    got_o, got_l = a.cpu().numpy().astype(np.float64), la.cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isneginf(got_l), np.isneginf(rl))
    fin = np.isfinite(rl)
    assert np.abs(got_l[fin] - rl[fin]).max(initial=0.0) <= 1e-5 * (1 + np.abs(rl[fin]).max(
        initial=0.0))
    assert np.abs(got_o - ro).max() <= 1e-5
    assert np.all(got_o[~fin] == 0.0)


@pytest.mark.parametrize("n", [8, 8 * 1001])
def test_accumulate_and_convert_are_exact(lib, n):
    """acc + bf16(part) is one fp32 addition per element, rounded the same way
    on both sides; the fp32 -> bf16 conversion rounds to nearest even."""
    import torch
    rng = np.random.default_rng(n)
    acc = rng.normal(size=n).astype(np.float32)
    part = torch.from_numpy(rng.normal(size=n).astype(np.float32)).bfloat16()
    want = acc + part.float().numpy()
    a = torch.from_numpy(acc).cuda()
    lib.accumulate_bf16(a, part.cuda())
    out = lib.convert_f32_bf16(a)
    torch.cuda.synchronize()
    assert np.array_equal(a.cpu().numpy(), want)
    # round to nearest even on the bit pattern: add 0x7FFF plus the kept lsb
    bits = want.view(np.uint32).astype(np.uint64)
    rne = ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16).astype(np.uint16)
    assert np.array_equal(out.cpu().view(torch.int16).numpy().view(np.uint16), rne)
