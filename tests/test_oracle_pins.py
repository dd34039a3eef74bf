"""Pins for the float64 oracle: each checks it against something other than itself.

A pin is a value the pages print, a closed form, an invariant of the
mathematics, an independent library routine or brute force.  Each test names
the plausible oracle mistake it would catch.
"""

import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest

from oracle import (
    attention_backward,
    attention_forward,
    dropout_keep,
    dropout_threshold,
    head_backward,
    philox4x32_10,
    philox_block,
    safe_softmax,
    valid_mask,
    weyl_constants,
)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# (causal, kv_len, block-mask kind) combinations used throughout
MASK_MODES = [
    dict(),
    dict(causal=True),
    dict(kv_len=True),
    dict(block=True),
    dict(causal=True, kv_len=True, block=True),
]


def _mask_args(mode, B, N, rng):
    causal = mode.get("causal", False)
    seqlens = None
    if mode.get("kv_len"):
        seqlens = rng.integers(max(1, N // 2), N + 1, size=B).astype(np.int32)
    block = None
    if mode.get("block"):
        nb = (N + 127) // 128
        block = (rng.random((nb, nb)) < 0.5).astype(np.uint8)
        np.fill_diagonal(block, 1)
    return causal, seqlens, block


def _rand(shape, rng):
    return rng.standard_normal(shape)


# ---------------------------------------------------------------------------
# Philox
# ---------------------------------------------------------------------------

def test_philox_round_structure_matches_numpy_philox4x64():
    """numpy.random.Philox is an independent Philox4x64-10.  The generic round
    function of the oracle at width 64 must reproduce its raw output (numpy
    increments the 256-bit counter before producing each 4-word block).  Catches
    a wrong permutation of the words, a wrong key schedule or round count."""
    rng = np.random.default_rng(5)
    for _ in range(20):
        ctr = [int(x) for x in rng.integers(0, 2**63, size=4, dtype=np.uint64)]
        ctr[1] = ctr[1] % 1000  # keep the carry into word 1 simple
        key = [int(x) for x in rng.integers(0, 2**63, size=2, dtype=np.uint64)]
        bg = np.random.Philox(counter=np.array(ctr, dtype=np.uint64),
                              key=np.array(key, dtype=np.uint64))
        got = [int(x) for x in bg.random_raw(4)]
        nxt = list(ctr)
        nxt[0] = (nxt[0] + 1) % 2**64
        if nxt[0] == 0:
            nxt[1] += 1
        want = list(philox_block(nxt, key, width=64, rounds=10))
        assert got == want


def test_weyl_constants_from_high_precision_arithmetic():
    """Key increments are floor(2^w (phi-1)) and floor(2^w (sqrt3-1)); recompute
    them with 60-digit decimal arithmetic (an independent route from isqrt)."""
    getcontext().prec = 60
    for w in (32, 64):
        s = Decimal(2) ** w
        phi1 = (Decimal(5).sqrt() - 1) / 2
        s31 = Decimal(3).sqrt() - 1
        assert weyl_constants(w) == (int(s * phi1), int(s * s31))


def test_philox4x32_vectorised_equals_scalar_definition():
    rng = np.random.default_rng(7)
    c = rng.integers(0, 2**32, size=(4, 64), dtype=np.uint64)
    k = rng.integers(0, 2**32, size=(2, 64), dtype=np.uint64)
    vec = philox4x32_10(c[0], c[1], c[2], c[3], k[0], k[1])
    for n in range(64):
        want = philox_block([c[i, n] for i in range(4)], [k[0, n], k[1, n]], 32, 10)
        assert tuple(int(v[n]) for v in vec) == want


def _curand_host_library():
    """cuRAND's shared library (host generators run on the CPU, no GPU needed)."""
    import ctypes
    import glob
    import sys
    pats = ["/usr/local/cuda/lib64/libcurand.so.10*", "/usr/local/cuda/lib64/libcurand.so*"]
    for p in sys.path:
        pats.append(os.path.join(p, "nvidia", "curand", "lib", "libcurand.so*"))
    for pat in pats:
        for path in sorted(glob.glob(pat)):
            try:
                return ctypes.CDLL(path)
            except OSError:
                continue
    return None


def curand_philox_words(seed, n):
    """The first n 32-bit outputs of cuRAND's host Philox4x32-10 generator
    (CURAND_RNG_PSEUDO_PHILOX4_32_10 = 161) seeded with `seed`, obtained by
    running the library; nothing of its internals is read."""
    import ctypes
    lib = _curand_host_library()
    if lib is None:
        pytest.skip("libcurand not found")
    gen = ctypes.c_void_p()
    assert lib.curandCreateGeneratorHost(ctypes.byref(gen), 161) == 0
    try:
        assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
        buf = (ctypes.c_uint32 * n)()
        assert lib.curandGenerate(gen, buf, ctypes.c_size_t(n)) == 0
        return [int(x) for x in buf]
    finally:
        lib.curandDestroyGenerator(gen)


@pytest.mark.parametrize("seed", [0, 1, 0xFFFFFFFF, 1 << 32, 0x0123456789ABCDEF,
                                  0x5EED000000000002, 0xDEADBEEFCAFEF00D,
                                  0xFFFFFFFFFFFFFFFF, 0x5EED0002])
def test_philox4x32_known_answers_from_curand(seed):
    """Known-answer pin of the 32-bit instance, multipliers included: cuRAND's
    host Philox4x32-10 generator is an independent implementation of the same
    published definition (Salmon et al., SC'11).  Seeded with s it uses key
    (s mod 2^32, s >> 32) and emits block k of its stream from counter
    (0, 0, k, 0) (layout found by experiment: block 0 at counter 0, later blocks
    step counter word 2).  A wrong digit in either multiplier, a swapped key
    word or a wrong Weyl step changes every word."""
    blocks = 16
    words = curand_philox_words(seed, 4 * blocks)
    key = [seed & 0xFFFFFFFF, seed >> 32]
    for k in range(blocks):
        assert tuple(words[4 * k:4 * k + 4]) == philox_block([0, 0, k, 0], key, 32, 10), k
    # the vectorised instance the dropout bits use gives the same words
    vec = philox4x32_10(0, 0, np.arange(blocks, dtype=np.uint64), 0, key[0], key[1])
    assert np.array_equal(np.stack(vec, axis=1).ravel(), np.array(words, dtype=np.uint32))


def test_philox4x32_words_are_uniform():
    """Chi-square of byte values and the mean of 2^20 words: a generator with a
    dropped round or a wrong multiplier on a structured counter sequence fails."""
    n = 1 << 18
    ctr = np.arange(n, dtype=np.uint64)
    words = np.stack(philox4x32_10(ctr, 0, 0, 0, 0x12345678, 0x9ABCDEF0)).ravel()
    assert abs(words.astype(np.float64).mean() / 2**32 - 0.5) < 5 * math.sqrt(1 / 12 / words.size)
    counts = np.bincount((words & 0xFF).astype(np.int64), minlength=256)
    e = words.size / 256
    chi2 = ((counts - e) ** 2 / e).sum()
    # 255 degrees of freedom: mean 255, sd ~22.6; allow 6 sd
    assert chi2 < 255 + 6 * math.sqrt(2 * 255)
    # successive counters must decorrelate: lag-1 correlation of the words
    x = words[::4].astype(np.float64)
    r = np.corrcoef(x[:-1], x[1:])[0, 1]
    assert abs(r) < 5 / math.sqrt(x.size)


# ---------------------------------------------------------------------------
# dropout bits
# ---------------------------------------------------------------------------

def test_dropout_threshold_is_exact_integer_of_float32_p():
    # 0.1 as float32 is 13421773 * 2^-27, so p * 2^16 = 6553.6000976... -> 6553
    assert dropout_threshold(0.1) == 6553
    assert dropout_threshold(0.0) == 0
    assert dropout_threshold(0.5) == 2**15
    assert dropout_threshold(np.nextafter(np.float32(1), np.float32(0))) == 2**16 - 1
    for bad in (-0.1, 1.0, 1.5, float("nan")):
        with pytest.raises(ValueError):
            dropout_threshold(bad)


def test_dropout_keep_uses_the_stated_counter_mapping():
    """keep(b,h,i,j) = 16-bit half (j & 1) of word ((j >> 1) & 3) of
    Philox4x32-10(counter=(j>>3, i, h, b), key=(seed lo, seed hi)) >= t,
    checked element by element by brute force."""
    seed = 0x0123456789ABCDEF
    p = 0.3
    t = dropout_threshold(p)
    rows = np.array([0, 1, 5, 130])
    keep = dropout_keep(seed, p, 3, 2, rows, 19)
    for a, i in enumerate(rows):
        for j in range(19):
            w = philox_block([j >> 3, int(i), 2, 3], [seed & 0xFFFFFFFF, seed >> 32])[(j >> 1) & 3]
            u = (w >> (16 * (j & 1))) & 0xFFFF
            assert keep[a, j] == (u >= t)


def test_dropout_keep_rate_within_5_sigma():
    """Over ~10^7 draws the keep fraction is 1 - t / 2^16 within 5 sigma
    (binomial), t = floor(p 2^16)."""
    for p in (0.1, 0.5):
        keep = dropout_keep(77, p, 1, 4, np.arange(2500), 4000)
        n = keep.size
        q = 1 - dropout_threshold(p) / 65536.0
        assert abs(keep.mean() - q) < 5 * math.sqrt(q * (1 - q) / n)


def test_dropout_scale_is_the_inverse_keep_probability():
    from oracle import dropout_scale
    assert dropout_scale(0.0) == 1.0
    assert dropout_scale(0.5) == 2.0
    assert dropout_scale(0.1) == 65536.0 / (65536.0 - 6553.0)


def test_dropout_p_zero_keeps_everything():
    assert dropout_keep(1, 0.0, 0, 0, np.arange(4), 9).all()


# ---------------------------------------------------------------------------
# softmax
# ---------------------------------------------------------------------------

def test_safe_softmax_pages_constant_rows():
    """The pages' overflow/underflow example: every score equal to c = +-20000.
    The safe softmax must give the uniform row with no inf/nan."""
    with open(os.path.join(GOLDEN, "safe_softmax_constant_rows.json")) as f:
        gold = json.load(f)
    for case in gold["cases"]:
        s = np.full((3, case["n"]), case["c"])
        p, lse, _, _ = safe_softmax(s, np.ones_like(s, dtype=bool))
        assert np.isfinite(p).all() and np.isfinite(lse).all()
        assert np.array_equal(p, np.full_like(p, case["p"]))
        assert np.allclose(lse, case["c"] + math.log(case["n"]), rtol=0, atol=1e-9)


def test_softmax_shift_invariance_at_plus_minus_20000():
    rng = np.random.default_rng(1)
    s = rng.standard_normal((16, 40))
    valid = rng.random((16, 40)) < 0.7
    valid[:, 0] = True
    p0, lse0, _, _ = safe_softmax(s, valid)
    for c in (20000.0, -20000.0):
        p, lse, _, _ = safe_softmax(s + c, valid)
        assert np.isfinite(p).all()
        assert np.abs(p - p0).max() < 1e-12
        assert np.abs(lse - (lse0 + c)).max() < 1e-9


def test_softmax_rows_sum_to_one_and_vanish_off_mask():
    rng = np.random.default_rng(2)
    for mode in MASK_MODES:
        B, N = 2, 300
        causal, seqlens, block = _mask_args(mode, B, N, rng)
        for b in range(B):
            kv = None if seqlens is None else seqlens[b]
            rows = np.arange(N)
            valid = valid_mask(N, rows, causal, kv, block)
            s = 3 * rng.standard_normal((N, N))
            p, _, _, _ = safe_softmax(s, valid)
            has = valid.any(axis=1)
            assert (p >= 0).all()
            assert np.abs(p.sum(axis=1)[has] - 1).max() < 1e-12
            assert (p[~valid] == 0).all()


def test_valid_mask_brute_force():
    rng = np.random.default_rng(3)
    N = 260
    block = (rng.random((3, 3)) < 0.5).astype(np.uint8)
    rows = np.arange(N)
    m = valid_mask(N, rows, True, 200, block)
    for i in range(0, N, 7):
        for j in range(0, N, 5):
            want = (j <= i) and (j < 200) and bool(block[i // 128, j // 128])
            assert m[i, j] == want


# ---------------------------------------------------------------------------
# forward: closed forms
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("mode", MASK_MODES)
def test_constant_v_rows_give_that_constant(mode):
    """V_j = v for every j gives O_i = v on every row with a valid key."""
    rng = np.random.default_rng(11)
    B, H, N, d = 2, 2, 200, 8
    causal, seqlens, block = _mask_args(mode, B, N, rng)
    q, k = _rand((B, H, N, d), rng), _rand((B, H, N, d), rng)
    vrow = rng.standard_normal((B, H, 1, d))
    v = np.broadcast_to(vrow, (B, H, N, d)).copy()
    o, lse = attention_forward(q, k, v, 0.3, causal, seqlens, block_mask=block)
    for b in range(B):
        kv = None if seqlens is None else seqlens[b]
        has = valid_mask(N, np.arange(N), causal, kv, block).any(axis=1)
        for h in range(H):
            assert np.abs(o[b, h][has] - vrow[b, h]).max() < 1e-12
            assert (o[b, h][~has] == 0).all()
            assert np.isneginf(lse[b, h][~has]).all()


@pytest.mark.parametrize("mode", MASK_MODES)
def test_zero_q_gives_masked_mean_and_log_count(mode):
    """Q = 0 makes every valid score 0: O_i is the mean of V over the valid keys
    of row i and LSE_i = ln(number of valid keys)."""
    rng = np.random.default_rng(12)
    B, H, N, d = 2, 1, 260, 4
    causal, seqlens, block = _mask_args(mode, B, N, rng)
    q = np.zeros((B, H, N, d))
    k, v = _rand((B, H, N, d), rng), _rand((B, H, N, d), rng)
    o, lse = attention_forward(q, k, v, 0.125, causal, seqlens, block_mask=block)
    for b in range(B):
        kv = None if seqlens is None else seqlens[b]
        valid = valid_mask(N, np.arange(N), causal, kv, block)
        for i in range(N):
            cnt = valid[i].sum()
            if cnt == 0:
                assert (o[b, 0, i] == 0).all() and np.isneginf(lse[b, 0, i])
                continue
            assert np.abs(o[b, 0, i] - v[b, 0][valid[i]].mean(axis=0)).max() < 1e-12
            assert abs(lse[b, 0, i] - math.log(cnt)) < 1e-12


def test_huge_scores_do_not_overflow_in_attention():
    """Scores of +-20000 through the whole forward: q = c e_0, every key e_0."""
    B, H, N, d = 1, 1, 6, 4
    k = np.zeros((B, H, N, d))
    k[..., 0] = 1.0
    v = np.arange(N * d, dtype=np.float64).reshape(1, 1, N, d)
    for c in (20000.0, -20000.0):
        q = np.zeros((B, H, N, d))
        q[..., 0] = c
        o, lse = attention_forward(q, k, v, 1.0)
        assert np.isfinite(o).all() and np.isfinite(lse).all()
        assert np.abs(o[0, 0] - v[0, 0].mean(axis=0)).max() < 1e-9
        assert np.abs(lse - (c + math.log(N))).max() < 1e-9


def test_slab_size_does_not_change_any_value():
    """Rows are independent: slabs of 1 row and of 256 rows agree to rounding
    (BLAS may sum in another order for another shape); the row-subset interface
    returns the same rows."""
    rng = np.random.default_rng(13)
    q, k, v = (_rand((1, 2, 300, 8), rng) for _ in range(3))
    a = attention_forward(q, k, v, 0.2, True, dropout_p=0.2, seed=9, slab=1)
    b = attention_forward(q, k, v, 0.2, True, dropout_p=0.2, seed=9, slab=256)
    assert np.abs(a[0] - b[0]).max() < 1e-13 and np.abs(a[1] - b[1]).max() < 1e-13
    rows = np.array([0, 131, 299])
    c = attention_forward(q, k, v, 0.2, True, dropout_p=0.2, seed=9, rows=rows)
    assert np.allclose(c[0], a[0][:, :, rows], rtol=0, atol=1e-14)


def test_dropout_is_unbiased_on_average():
    """E[Z/(1-p)] = 1: averaged over many seeds, dropped attention approaches
    the undropped output (inverted dropout)."""
    rng = np.random.default_rng(14)
    q, k, v = (_rand((1, 1, 16, 4), rng) for _ in range(3))
    o0, lse0 = attention_forward(q, k, v, 0.5)
    acc = np.zeros_like(o0)
    n = 400
    for s in range(n):
        o, lse = attention_forward(q, k, v, 0.5, dropout_p=0.25, seed=1000 + s)
        assert np.array_equal(lse, lse0)  # LSE is that of the undropped softmax
        acc += o
    err = np.abs(acc / n - o0).max()
    assert err < 0.15


# ---------------------------------------------------------------------------
# forward + backward against an independent library routine
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("mode", MASK_MODES)
def test_matches_torch_sdpa_and_autograd_without_dropout(mode):
    """torch.nn.functional.scaled_dot_product_attention (CPU, float64, boolean
    mask) and torch.autograd compute the same definition independently."""
    import torch

    rng = np.random.default_rng(15)
    B, H, N, d = 2, 2, 150, 16
    causal, seqlens, block = _mask_args(mode, B, N, rng)
    q, k, v, do = (_rand((B, H, N, d), rng) for _ in range(4))
    scale = 0.2
    o, lse = attention_forward(q, k, v, scale, causal, seqlens, block_mask=block)
    dq, dk, dv = attention_backward(q, k, v, do, scale, causal, seqlens, block_mask=block)

    mask = np.stack([valid_mask(N, np.arange(N), causal,
                                None if seqlens is None else seqlens[b], block)
                     for b in range(B)])[:, None]
    has = mask.any(axis=-1)  # rows with at least one valid key
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=torch.tensor(mask), scale=scale)
    # fully masked rows give NaN in SDPA; compare only rows that have keys
    to = torch.where(torch.tensor(has)[..., None], to, torch.zeros_like(to))
    (to * torch.tensor(do)).sum().backward()
    assert np.abs(o - to.detach().numpy()).max() < 1e-12
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.abs(mine - ref.numpy()).max() < 1e-10
    # the LSE against a direct logsumexp of the masked scores
    s = scale * np.einsum("bhid,bhjd->bhij", q, k)
    s = np.where(mask, s, -np.inf)
    with np.errstate(divide="ignore"):
        ref_lse = np.log(np.exp(s - s.max(-1, keepdims=True, initial=-1e300)).sum(-1)) \
            + s.max(-1, initial=-1e300)
    assert np.abs(np.where(has, lse - ref_lse, 0)).max() < 1e-12


# ---------------------------------------------------------------------------
# backward: finite differences and identities
# ---------------------------------------------------------------------------

FD_CASES = [
    (5, 4, dict(), 0.0),
    (8, 8, dict(causal=True), 0.0),
    (16, 4, dict(kv_len=True), 0.0),
    (16, 8, dict(causal=True, kv_len=True), 0.3),
    (8, 4, dict(), 0.5),
]


@pytest.mark.parametrize("N,d,mode,p", FD_CASES)
def test_backward_matches_central_finite_differences(N, d, mode, p):
    """dL/dx for L = sum(O * dO) by central differences in float64, dropout bits
    held fixed by the seed: catches a dropped term, sign or transposition."""
    rng = np.random.default_rng(100 + N + d)
    B, H = 1, 1
    causal = mode.get("causal", False)
    seqlens = np.array([max(1, N - 3)], dtype=np.int32) if mode.get("kv_len") else None
    q, k, v, do = (_rand((B, H, N, d), rng) for _ in range(4))
    scale, seed = 0.7, 4242

    def loss(q_, k_, v_):
        o, _ = attention_forward(q_, k_, v_, scale, causal, seqlens, p, seed)
        return float((o * do).sum())

    dq, dk, dv = attention_backward(q, k, v, do, scale, causal, seqlens, p, seed)
    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        err = np.linalg.norm(num - g) / max(np.linalg.norm(num), 1e-30)
        assert err < 1e-6, (name, err)


@pytest.mark.parametrize("p", [0.0, 0.2])
def test_backward_identities(p):
    """(i) sum_j dK_j = 0 per (b,h); (ii) D_i = sum_j P_ij dP_ij equals
    sum_c dO_ic O_ic; (iii) constant key rows give dQ = 0."""
    rng = np.random.default_rng(21)
    N, d = 200, 8
    q, k, v, do = (_rand((N, d), rng) for _ in range(4))
    keep = dropout_keep(5, p, 0, 0, np.arange(N), N) if p > 0 else None
    dq, dk, dv, dsum = head_backward(q, k, v, do, 0.4, True, None, None, keep, p)
    assert np.abs(dk.sum(axis=0)).max() < 1e-10
    o, _ = attention_forward(q[None, None], k[None, None], v[None, None], 0.4, True,
                             dropout_p=p, seed=5)
    assert np.abs(dsum - (do * o[0, 0]).sum(axis=1)).max() < 1e-10
    kc = np.broadcast_to(k[:1], k.shape).copy()
    dq2, _, _, _ = head_backward(q, kc, v, do, 0.4, True, None, None, keep, p)
    assert np.abs(dq2).max() < 1e-12


def test_zero_q_gives_closed_form_dv():
    """Q = 0, no dropout: P_ij = 1/n_i on the valid keys, so
    dV_j = sum over rows i where j is valid of dO_i / n_i."""
    rng = np.random.default_rng(22)
    N, d = 140, 4
    q = np.zeros((N, d))
    k, v, do = (_rand((N, d), rng) for _ in range(3))
    _, _, dv, _ = head_backward(q, k, v, do, 1.0, True, 100)
    valid = valid_mask(N, np.arange(N), True, 100)
    n = valid.sum(axis=1)
    want = np.zeros((N, d))
    for i in range(N):
        for j in np.nonzero(valid[i])[0]:
            want[j] += do[i] / n[i]
    assert np.abs(dv - want).max() < 1e-12


@pytest.mark.parametrize("mode", MASK_MODES)
def test_sampled_backward_matches_torch_autograd(mode):
    """The row- and column-sampled backward (used to check full-size runs)
    against torch autograd through SDPA, with the same masks, no dropout."""
    import torch

    from oracle import head_backward_cols, head_backward_rows, head_forward_rows

    rng = np.random.default_rng(31)
    B, N, d = 1, 300, 8
    causal, seqlens, block = _mask_args(mode, B, N, rng)
    kv = None if seqlens is None else int(seqlens[0])
    q, k, v, do = (_rand((N, d), rng) for _ in range(4))
    mask = valid_mask(N, np.arange(N), causal, kv, block)
    has = mask.any(axis=1)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(
        tq[None], tk[None], tv[None], attn_mask=torch.tensor(mask)[None], scale=0.3)[0]
    to = torch.where(torch.tensor(has)[:, None], to, torch.zeros_like(to))
    (to * torch.tensor(do)).sum().backward()
    rows = np.array([0, 5, 127, 128, 299])
    cols = np.array([0, 3, 128, 250, 299])
    dq = head_backward_rows(q, k, v, do, 0.3, rows, causal, kv, block)
    dk, dv = head_backward_cols(q, k, v, do, 0.3, cols, causal, kv, block, slab=64)
    o_rows, _ = head_forward_rows(q, k, v, 0.3, rows, causal, kv, block)
    assert np.abs(o_rows - to.detach().numpy()[rows]).max() < 1e-12
    assert np.abs(dq - tq.grad.numpy()[rows]).max() < 1e-10
    assert np.abs(dk - tk.grad.numpy()[cols]).max() < 1e-10
    assert np.abs(dv - tv.grad.numpy()[cols]).max() < 1e-10


def test_sampled_forward_rows_use_the_head_own_dropout_bits():
    """head_forward_rows(b, h) equals the (b, h) slice of the batched forward."""
    from oracle import head_forward_rows

    rng = np.random.default_rng(33)
    q, k, v = (_rand((2, 3, 140, 4), rng) for _ in range(3))
    o, lse = attention_forward(q, k, v, 0.4, True, dropout_p=0.2, seed=5)
    rows = np.array([0, 64, 139])
    for b, h in ((0, 0), (1, 2)):
        ro, rl = head_forward_rows(q[b, h], k[b, h], v[b, h], 0.4, rows, True,
                                   dropout_p=0.2, seed=5, b=b, h=h)
        assert np.abs(ro - o[b, h][rows]).max() < 1e-12
        assert np.abs(rl - lse[b, h][rows]).max() < 1e-12


def test_sampled_backward_with_dropout_matches_finite_differences():
    """With dropout (bits fixed by the seed), sampled dQ rows and dK / dV
    columns against central differences of L = sum(O * dO)."""
    from oracle import head_backward_cols, head_backward_rows

    rng = np.random.default_rng(32)
    N, d, p, seed = 12, 4, 0.3, 77
    q, k, v, do = (_rand((1, 1, N, d), rng) for _ in range(4))

    def loss(q_, k_, v_):
        o, _ = attention_forward(q_, k_, v_, 0.5, True, None, p, seed)
        return float((o * do).sum())

    eps = 1e-6
    rows, cols = np.array([1, 7, 11]), np.array([0, 6, 10])
    dq = head_backward_rows(q[0, 0], k[0, 0], v[0, 0], do[0, 0], 0.5, rows, True,
                            dropout_p=p, seed=seed)
    dk, dv = head_backward_cols(q[0, 0], k[0, 0], v[0, 0], do[0, 0], 0.5, cols, True,
                                dropout_p=p, seed=seed, slab=5)
    for name, x, sel, g in (("q", q, rows, dq), ("k", k, cols, dk), ("v", v, cols, dv)):
        num = np.zeros((sel.size, d))
        for a, r in enumerate(sel):
            for c in range(d):
                xp, xm = x.copy(), x.copy()
                xp[0, 0, r, c] += eps
                xm[0, 0, r, c] -= eps
                args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
                args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
                num[a, c] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        assert np.linalg.norm(num - g) / np.linalg.norm(num) < 1e-6, name


# ---------------------------------------------------------------------------
# N_q != N_k (bottom-right causal alignment) and packed variable-length batches
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("nq,nk", [(3, 7), (7, 3), (5, 5), (1, 9), (9, 1), (130, 260)])
def test_bottom_right_causal_mask_brute_force(nq, nk):
    """Query i sees key j iff j <= i + nk - nq: written as plain loops; a
    top-left alignment or an off-by-one in the offset fails."""
    got = valid_mask(nk, np.arange(nq), True, None, None, n_q=nq)
    for i in range(nq):
        for j in range(nk):
            assert got[i, j] == (j - i <= nk - nq)


@pytest.mark.parametrize("nq,nk,kv", [(40, 100, None), (100, 40, None), (64, 200, 150),
                                      (200, 64, 50), (1, 33, None)])
def test_bottom_right_causal_matches_torch_lower_right(nq, nk, kv):
    """torch's causal_lower_right bias is an independent definition of the
    bottom-right alignment: SDPA with it (and autograd) must give the oracle's
    O and gradients on every row that has a key (rows without one: O = 0,
    LSE = -inf, no gradient)."""
    import torch
    from torch.nn.attention.bias import causal_lower_right

    rng = np.random.default_rng(nq * 7 + nk)
    H, d = 2, 8
    q, do = _rand((1, H, nq, d), rng), _rand((1, H, nq, d), rng)
    k, v = _rand((1, H, nk, d), rng), _rand((1, H, nk, d), rng)
    seq = None if kv is None else np.array([kv], dtype=np.int32)
    o, lse = attention_forward(q, k, v, 0.3, True, seq)
    dq, dk, dv = attention_backward(q, k, v, do, 0.3, True, seq)
    mask = causal_lower_right(nq, nk)._materialize(torch.device("cpu"))
    if kv is not None:
        mask = mask & (torch.arange(nk) < kv)[None, :]
    has = mask.any(dim=-1).numpy()
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=0.3)
    to = torch.where(torch.tensor(has)[:, None], to, torch.zeros_like(to))
    (to * torch.tensor(do)).sum().backward()
    assert np.abs(o - to.detach().numpy()).max() < 1e-12
    assert (o[:, :, ~has] == 0).all() and np.isneginf(lse[:, :, ~has]).all()
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.abs(mine - ref.numpy()).max() < 1e-10


@pytest.mark.parametrize("nq,nk", [(50, 130), (130, 50)])
def test_zero_q_bottom_right_closed_form(nq, nk):
    """Q = 0 under the bottom-right causal mask: row i has
    n_i = clip(i + nk - nq + 1, 0, nk) valid keys, the first n_i of them, so
    O_i = mean(V_0 .. V_{n_i - 1}) and LSE_i = ln n_i (n_i = 0: O = 0, -inf)."""
    rng = np.random.default_rng(41)
    d = 4
    q = np.zeros((1, 1, nq, d))
    k, v = _rand((1, 1, nk, d), rng), _rand((1, 1, nk, d), rng)
    o, lse = attention_forward(q, k, v, 0.5, True)
    for i in range(nq):
        n = min(max(i + nk - nq + 1, 0), nk)
        if n == 0:
            assert (o[0, 0, i] == 0).all() and np.isneginf(lse[0, 0, i])
        else:
            assert np.abs(o[0, 0, i] - v[0, 0, :n].mean(axis=0)).max() < 1e-12
            assert abs(lse[0, 0, i] - math.log(n)) < 1e-12


def _pack(seqs):
    """[B] list of [H, n_b, d] arrays -> packed [sum n_b, H, d] and offsets."""
    cu = np.concatenate([[0], np.cumsum([s.shape[1] for s in seqs])]).astype(np.int32)
    packed = np.concatenate([s.transpose(1, 0, 2) for s in seqs], axis=0)
    return packed, cu


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_each_sequence_on_its_own(causal):
    """Packed sequences (lengths 0, 1, 129, 300, 77 queries against other key
    counts) give, row for row, the padded oracle run on each sequence alone
    (no dropout: the padded call would number the sequence 0).  Catches wrong
    offsets, a token / head transposition or attention leaking across
    sequences."""
    from oracle import attention_forward_varlen, attention_backward_varlen
    rng = np.random.default_rng(51)
    H, d, scale = 2, 8, 0.35
    lq = [0, 1, 129, 300, 77]
    lk = [5, 1, 200, 300, 31]
    qs = [_rand((H, n, d), rng) for n in lq]
    dos = [_rand((H, n, d), rng) for n in lq]
    ks = [_rand((H, n, d), rng) for n in lk]
    vs = [_rand((H, n, d), rng) for n in lk]
    q, cu_q = _pack(qs)
    do, _ = _pack(dos)
    k, cu_k = _pack(ks)
    v, _ = _pack(vs)
    o, lse = attention_forward_varlen(q, k, v, cu_q, cu_k, scale, causal)
    dq, dk, dv = attention_backward_varlen(q, k, v, do, cu_q, cu_k, scale, causal)
    for b in range(len(lq)):
        if lq[b] == 0:
            continue
        ro, rl = attention_forward(qs[b][None], ks[b][None], vs[b][None], scale, causal)
        rg = attention_backward(qs[b][None], ks[b][None], vs[b][None], dos[b][None], scale,
                                causal)
        sq = slice(cu_q[b], cu_q[b + 1])
        sk = slice(cu_k[b], cu_k[b + 1])
        # equal up to BLAS summation order (strided vs contiguous operands)
        assert np.abs(o[sq].transpose(1, 0, 2) - ro[0]).max() < 1e-12
        empty = np.isneginf(rl[0])
        assert np.array_equal(np.isneginf(lse[:, sq]), empty)
        assert np.abs(np.where(empty, 0.0, lse[:, sq] - np.where(empty, 0.0, rl[0]))).max() < 1e-12
        assert np.abs(dq[sq].transpose(1, 0, 2) - rg[0][0]).max() < 1e-10
        assert np.abs(dk[sk].transpose(1, 0, 2) - rg[1][0]).max() < 1e-10
        assert np.abs(dv[sk].transpose(1, 0, 2) - rg[2][0]).max() < 1e-10


def test_varlen_dropout_and_key_lengths_use_the_sequence_index():
    """With dropout the keep bits of sequence b are those of batch entry b:
    packed sequences of equal query and key length equal a padded batch whose
    entry b holds sequence b at its start, the rest masked by key lengths."""
    from oracle import attention_forward_varlen, attention_backward_varlen
    rng = np.random.default_rng(52)
    H, d, N, p, seed = 2, 8, 140, 0.25, 99
    lens = [140, 60, 131]
    full = [_rand((4, H, N, d), rng) for _ in range(len(lens))]  # q, k, v, dO per sequence
    seqs = [[f[x][:, :n] for f, n in zip(full, lens)] for x in range(4)]
    q, cu = _pack(seqs[0])
    k, _ = _pack(seqs[1])
    v, _ = _pack(seqs[2])
    do, _ = _pack(seqs[3])
    pq, pk, pv, pdo = (np.stack([f[x] for f in full]) for x in range(4))
    seqlens = np.array(lens, dtype=np.int32)
    for causal in (False, True):
        o, lse = attention_forward_varlen(q, k, v, cu, cu, 0.3, causal, None, p, seed)
        dq, dk, dv = attention_backward_varlen(q, k, v, do, cu, cu, 0.3, causal, None, p, seed)
        ro, rl = attention_forward(pq, pk, pv, 0.3, causal, seqlens, p, seed)
        rdq, rdk, rdv = attention_backward(pq, pk, pv, pdo, 0.3, causal, seqlens, p, seed)
        for b, n in enumerate(lens):
            s = slice(cu[b], cu[b + 1])
            # padded rows of the padded batch only add masked keys (and, for
            # causal, N = N_k keeps the alignment), so rows i < n agree
            assert np.abs(o[s].transpose(1, 0, 2) - ro[b][:, :n]).max() < 1e-12
            assert np.abs(lse[:, s] - rl[b][:, :n]).max() < 1e-12
            # dK, dV of keys j < n: the padded batch's extra query rows i >= n
            # see those keys too (key padding masks keys, not queries), so
            # only dQ rows are comparable
            assert np.abs(dq[s].transpose(1, 0, 2) - rdq[b][:, :n]).max() < 1e-10
    # key lengths inside packed sequences: keys past seqlens_k[b] are masked
    o1, _ = attention_forward_varlen(q, k, v, cu, cu, 0.3, False, np.array([10, 60, 20]))
    o2, _ = attention_forward_varlen(q, k, v, cu, cu, 0.3, False, None)
    assert np.array_equal(o1[cu[1]:cu[2]], o2[cu[1]:cu[2]])       # 60 = the full length
    assert not np.allclose(o1[cu[0]:cu[1]], o2[cu[0]:cu[1]])


def test_varlen_backward_matches_finite_differences():
    """Packed backward (bottom-right causal, dropout, a key length) against
    central differences of L = sum(O * dO)."""
    from oracle import attention_forward_varlen, attention_backward_varlen
    rng = np.random.default_rng(53)
    H, d, p, seed = 1, 3, 0.3, 5
    cu_q = np.array([0, 4, 4, 9], dtype=np.int32)
    cu_k = np.array([0, 6, 8, 11], dtype=np.int32)
    skl = np.array([5, 2, 3], dtype=np.int32)
    q, do = _rand((9, H, d), rng), _rand((9, H, d), rng)
    k, v = _rand((11, H, d), rng), _rand((11, H, d), rng)

    def loss(q_, k_, v_):
        o, _ = attention_forward_varlen(q_, k_, v_, cu_q, cu_k, 0.6, True, skl, p, seed)
        return float((o * do).sum())

    grads = attention_backward_varlen(q, k, v, do, cu_q, cu_k, 0.6, True, skl, p, seed)
    eps = 1e-6
    for name, x, g in zip("qkv", (q, k, v), grads):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            a = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            num[idx] = (loss(*a) - loss(*m)) / (2 * eps)
        err = np.linalg.norm(num - g) / max(np.linalg.norm(num), 1e-30)
        assert err < 1e-6, (name, err)


# ---------------------------------------------------------------------------
# merging partial results over disjoint key sets (context parallelism)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_merge_of_key_blocks_equals_attention_over_all_keys(causal):
    """Attention of Q against key blocks 0..3 taken apart (each block's own
    (O, LSE), causal only on the diagonal block, blocks past it skipped) and
    merged left to right equals attention over all keys: the decomposition a
    context-parallel ring computes.  A wrong weight (no renormalisation, a
    missing exp) or a mishandled empty block fails."""
    from oracle import merge_partials
    rng = np.random.default_rng(61)
    W, n, d = 4, 50, 8
    q, k, v = (_rand((1, 2, W * n, d), rng) for _ in range(3))
    o_full, l_full = attention_forward(q, k, v, 0.4, causal)
    for r in range(W):  # query block r
        qr = q[:, :, r * n:(r + 1) * n]
        o = np.zeros_like(qr)
        lse = np.full(qr.shape[:-1], -np.inf)
        for c in range(W):  # key block c
            if causal and c > r:
                continue
            kc, vc = k[:, :, c * n:(c + 1) * n], v[:, :, c * n:(c + 1) * n]
            op, lp = attention_forward(qr, kc, vc, 0.4, causal and c == r)
            o, lse = merge_partials(o, lse, op, lp)
        assert np.abs(o - o_full[:, :, r * n:(r + 1) * n]).max() < 1e-12
        assert np.abs(lse - l_full[:, :, r * n:(r + 1) * n]).max() < 1e-12


def test_merge_with_empty_parts():
    """Empty parts (LSE = -inf) change nothing; two empty parts stay empty."""
    from oracle import merge_partials
    rng = np.random.default_rng(62)
    o = rng.standard_normal((5, 4))
    lse = rng.standard_normal(5)
    inf = np.full(5, -np.inf)
    o2, l2 = merge_partials(o, lse, np.zeros((5, 4)), inf)
    assert np.array_equal(o2, o) and np.array_equal(l2, lse)
    o3, l3 = merge_partials(np.ones((5, 4)), inf, o, lse)
    assert np.array_equal(o3, o) and np.array_equal(l3, lse)
    o4, l4 = merge_partials(np.ones((5, 4)), inf, np.ones((5, 4)), inf)
    assert (o4 == 0).all() and np.isneginf(l4).all()


@pytest.mark.parametrize("causal,p", [(False, 0.0), (True, 0.0), (False, 0.2), (True, 0.3)])
def test_block_backward_sums_to_the_full_backward(causal, p):
    """The per-key-block backward given the full rows' LSE and D, summed over
    blocks (query blocks x key blocks), equals the full backward: the
    decomposition a context-parallel ring uses, with dropout too (each block
    keys its bits by the rows' and keys' positions in the sequence).  Dropping
    the D term, using the block's own LSE, a wrong causal offset or bits keyed
    by positions inside the block fails."""
    from oracle import attention_backward, head_backward_block
    rng = np.random.default_rng(63)
    W, n, d, scale, seed = 3, 40, 8, 0.45, 0x5EED
    N = W * n
    q, k, v, do = (_rand((N, d), rng) for _ in range(4))
    o, lse = attention_forward(q[None, None], k[None, None], v[None, None], scale, causal,
                               dropout_p=p, seed=seed)
    full = attention_backward(q[None, None], k[None, None], v[None, None], do[None, None], scale,
                              causal, None, p, seed)
    dq, dk, dv = (x[0, 0] for x in full)
    delta = (do * o[0, 0]).sum(axis=1)
    gq, gk, gv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for r in range(W):
        rs = slice(r * n, (r + 1) * n)
        for c in range(W):
            cs = slice(c * n, (c + 1) * n)
            a, b, e = head_backward_block(q[rs], k[cs], v[cs], do[rs], lse[0, 0, rs], delta[rs],
                                          scale, causal, N, N, r * n, c * n, p, seed)
            gq[rs] += a
            gk[cs] += b
            gv[cs] += e
    assert np.abs(gq - dq).max() < 1e-10
    assert np.abs(gk - dk).max() < 1e-10
    assert np.abs(gv - dv).max() < 1e-10


# ---------------------------------------------------------------------------
# QKV projection (the layer in front of attention)
# ---------------------------------------------------------------------------

def test_qkv_projection_brute_force():
    """Every output element as an explicit sum over the model dimension, with
    the stated column / token mapping written out as loops."""
    from oracle import qkv_projection
    rng = np.random.default_rng(91)
    B, N, H, d, Dm = 2, 3, 2, 4, 5
    x = rng.standard_normal((B * N, Dm))
    w = rng.standard_normal((3 * H * d, Dm))
    bias = rng.standard_normal(3 * H * d)
    q, k, v = qkv_projection(x, w, bias, B, H, d)
    for which, out in enumerate((q, k, v)):
        for b in range(B):
            for h in range(H):
                for n in range(N):
                    for e in range(d):
                        c = which * H * d + h * d + e
                        want = sum(x[b * N + n, f] * w[c, f] for f in range(Dm)) + bias[c]
                        assert abs(out[b, h, n, e] - want) < 1e-12


def test_qkv_projection_matches_torch_linear():
    """torch.nn.functional.linear, split into q, k, v and heads with
    view / permute: an independent route to the same tensors."""
    import torch
    from oracle import qkv_projection
    rng = np.random.default_rng(92)
    B, N, H, d, Dm = 3, 17, 4, 8, 24
    x = rng.standard_normal((B * N, Dm))
    w = rng.standard_normal((3 * H * d, Dm))
    bias = rng.standard_normal(3 * H * d)
    q, k, v = qkv_projection(x, w, bias, B, H, d)
    y = torch.nn.functional.linear(torch.tensor(x), torch.tensor(w), torch.tensor(bias))
    ref = y.view(B, N, 3, H, d).permute(2, 0, 3, 1, 4)
    for i, got in enumerate((q, k, v)):
        assert np.abs(got - ref[i].numpy()).max() < 1e-12
    q0, _, _ = qkv_projection(x, w, None, B, H, d)
    assert np.abs(q0 - (q - bias[:H * d].reshape(1, H, 1, d))).max() < 1e-12


# ---------------------------------------------------------------------------
# sequence offsets of a slice (dropout bits keyed by the absolute (i, j))
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("key0", [0, 5, 13, 256, 4001])
def test_dropout_keep_with_key_offset_is_the_slice_of_the_whole_row(key0):
    """Keys key0 .. key0 + n - 1 take the bits those keys have in the whole
    row, for block-aligned and unaligned offsets alike."""
    from oracle import dropout_keep
    rows = np.array([0, 7, 1000, 123457])
    n = 37
    whole = dropout_keep(99, 0.3, 2, 5, rows, key0 + n)
    assert np.array_equal(dropout_keep(99, 0.3, 2, 5, rows, n, key0=key0), whole[:, key0:])


def test_row_and_column_helpers_on_a_diagonal_slice_match_the_whole_problem():
    """Under a block mask that keeps only the diagonal 128 x 128 blocks, a
    query tile sees only its own key tile: the helpers on that slice, told its
    sequence offsets, give the whole problem's rows and columns (dropout on)."""
    from oracle.attention_ref import head_backward_cols, head_backward_rows, head_forward_rows
    rng = np.random.default_rng(4)
    N, d, t = 384, 16, 2
    q, k, v, do = (rng.standard_normal((N, d)) for _ in range(4))
    bm = np.eye(N // 128, dtype=np.uint8)
    kw = dict(dropout_p=0.2, seed=17, b=1, h=3)
    rows = np.array([0, 5, 127])
    sl = slice(128 * t, 128 * t + 128)
    full_o, full_l = head_forward_rows(q, k, v, 0.25, rows + 128 * t, block_mask=bm, **kw)
    part_o, part_l = head_forward_rows(q[sl], k[sl], v[sl], 0.25, rows, row0=128 * t,
                                       key0=128 * t, **kw)
    assert np.allclose(full_o, part_o, rtol=0, atol=1e-12)
    assert np.allclose(full_l, part_l, rtol=0, atol=1e-12)
    full_dq = head_backward_rows(q, k, v, do, 0.25, rows + 128 * t, block_mask=bm, **kw)
    part_dq = head_backward_rows(q[sl], k[sl], v[sl], do[sl], 0.25, rows, row0=128 * t,
                                 key0=128 * t, **kw)
    assert np.allclose(full_dq, part_dq, rtol=0, atol=1e-12)
    cols = np.array([1, 64, 126])
    full_dk, full_dv = head_backward_cols(q, k, v, do, 0.25, cols + 128 * t, block_mask=bm, **kw)
    part_dk, part_dv = head_backward_cols(q[sl], k[sl], v[sl], do[sl], 0.25, cols,
                                          row0=128 * t, key0=128 * t, **kw)
    assert np.allclose(full_dk, part_dk, rtol=0, atol=1e-12)
    assert np.allclose(full_dv, part_dv, rtol=0, atol=1e-12)
    # the offsets matter: without them the dropout bits are another draw
    wrong_o, _ = head_forward_rows(q[sl], k[sl], v[sl], 0.25, rows, **kw)
    assert not np.allclose(full_o, wrong_o, rtol=0, atol=1e-6)


# ---------------------------------------------------------------------------
# grouped K / V heads
# ---------------------------------------------------------------------------

def test_gqa_forward_uses_the_group_head():
    """Without dropout each query head's O and LSE are plain attention against
    K / V head h // G, evaluated head by head; the mapping h % H_kv (or any
    other) gives different outputs."""
    from oracle import attention_forward_gqa
    rng = np.random.default_rng(77)
    B, H, Hkv, N, d = 2, 6, 2, 9, 4
    q = _rand((B, H, N, d), rng)
    k, v = _rand((B, Hkv, N, d), rng), _rand((B, Hkv, N, d), rng)
    o, lse = attention_forward_gqa(q, k, v, 0.4, True)
    G = H // Hkv
    for h in range(H):
        oh, lh = attention_forward(q[:, h:h + 1], k[:, h // G:h // G + 1], v[:, h // G:h // G + 1],
                                   0.4, True)
        assert np.abs(o[:, h:h + 1] - oh).max() < 1e-12
        assert np.abs(lse[:, h:h + 1] - lh).max() < 1e-12
    wrong, _ = attention_forward(q[:, 1:2], k[:, 1:2], v[:, 1:2], 0.4, True)  # h % H_kv
    assert np.abs(o[:, 1:2] - wrong).max() > 1e-3


def test_gqa_backward_matches_finite_differences():
    """dQ and the shared heads' dK, dV (sums over each group) against central
    differences of L = sum(O * dO), with a causal mask and dropout."""
    from oracle import attention_backward_gqa, attention_forward_gqa
    rng = np.random.default_rng(78)
    B, H, Hkv, N, d, p, seed = 1, 4, 2, 6, 3, 0.3, 11
    q, do = _rand((B, H, N, d), rng), _rand((B, H, N, d), rng)
    k, v = _rand((B, Hkv, N, d), rng), _rand((B, Hkv, N, d), rng)

    def loss(q_, k_, v_):
        o, _ = attention_forward_gqa(q_, k_, v_, 0.7, True, None, p, seed)
        return float((o * do).sum())

    grads = attention_backward_gqa(q, k, v, do, 0.7, True, None, p, seed)
    assert grads[1].shape == k.shape and grads[2].shape == v.shape
    eps = 1e-6
    for name, x, g in zip("qkv", (q, k, v), grads):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            a = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            num[idx] = (loss(*a) - loss(*m)) / (2 * eps)
        err = np.linalg.norm(num - g) / max(np.linalg.norm(num), 1e-30)
        assert err < 1e-6, (name, err)
