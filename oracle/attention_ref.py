"""Standard (materialising) softmax attention in float64: the oracle.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this module.  It shares
no code with the CUDA path and never receives a value computed by it.

What it computes, and where that is defined
-------------------------------------------
The method (FlashAttention) is *exact*: it returns the same result as standard
attention and differs only in how it moves data (researchpapers.dev
"FlashAttention 详解:IO 感知精确注意力,提速 2-4 倍", sections "快速答案" and the
FAQ entry asking whether it is exact or approximate).  So this oracle is the
textbook definition written out, one (batch, head) at a time, materialising the
full score matrix exactly as the "standard attention" the pages describe
(suanlizi.com FlashAttention summary, sections "核心操作融合" and "分块计算"):

    S = scale * Q K^T                   score matrix, N x N
    P = softmax over the valid keys     row-wise, safe form (subtract the row max)
    O = dropout(P) V

and the backward is the plain chain rule through those three steps.  The safe
softmax (subtracting the row maximum before exp) is the form the pages require
to avoid overflow at scores like +20000 and a vanishing denominator at -20000
(llm-deploy "tensorrt-llm/flash-attention.md", safe-softmax section on
上溢出 / 下溢出).  The saved statistic is the per-row log-sum-exp
LSE = m + ln(l), the (m, l) pair of the online softmax collapsed to one number
(same page, closing "解决方案" paragraph, whose symbol list is garbled; the
running max m and row sum l are the readings used here).

Readings taken where the pages are silent:
  * scale is a caller-given float applied to Q K^T before masking and the max;
  * causal: query i may attend key j iff j <= i + (N_k - N_q) (0-based; the
    last query is aligned with the last key, "bottom-right"; with N_q = N_k
    this is j <= i).  When N_q > N_k the first N_q - N_k queries see no key.
    Key padding does not move the alignment: N_k is the key count of the
    layout (or of the packed sequence), not the padded length;
  * key padding: per-batch length L_b, keys j >= L_b are invalid; query rows
    are not masked (they still attend the valid keys);
  * block mask: uint8 [ceil(N/128)]^2 shared by all (b, h); entry 0 removes the
    whole 128 x 128 block of (query, key) pairs;
  * all masks combine by logical AND;
  * a row with no valid key has P = 0, O = 0 and LSE = -inf;
  * dropout is inverted dropout on the normalised P: P_drop = P * Z / q with
    q = 1 - t / 2^16 the keep probability of the generator below, Z the keep
    bit; LSE is that of the undropped softmax;
  * keep bit Z(b,h,i,j): one Philox4x32-10 block serves eight consecutive
    keys: key (seed mod 2^32, seed >> 32), counter (j >> 3, i, h, b); key j
    takes the 16-bit half (j & 1) (0 = low) of output word ((j >> 1) & 3);
    keep iff that 16-bit value >= t with t = min(floor(p * 2^16), 2^16 - 1),
    p the float32 value the library receives.  The realised drop probability
    is therefore t / 2^16 (0.0999908 for p = 0.1).

Parity pins for every function here live in ``tests/test_oracle_pins.py``.
"""

from __future__ import annotations

import math

import numpy as np

from .philox_ref import philox4x32_10

BLOCK = 128  # block-mask granularity (128 x 128 blocks of (query, key) pairs)


# ----------------------------------------------------------------------------
# masks and dropout bits
# ----------------------------------------------------------------------------

def valid_mask(n, rows, causal=False, kv_len=None, block_mask=None, n_q=None):
    """Boolean [len(rows), n]: which (query i, key j) pairs take part.

    n: number of keys.  rows: query indices (int array).  kv_len: valid key
    count for this batch entry (None = n).  block_mask: uint8 [nbq, nbk] or
    None.  n_q: number of queries (None = n); under the causal mask query i
    sees key j iff j <= i + (n - n_q).
    """
    rows = np.asarray(rows, dtype=np.int64)
    i = rows[:, None]
    j = np.arange(n, dtype=np.int64)[None, :]
    ok = np.ones((rows.size, n), dtype=bool)
    if kv_len is not None:
        ok &= j < int(kv_len)
    if causal:
        off = 0 if n_q is None else int(n) - int(n_q)
        ok &= j <= i + off
    if block_mask is not None:
        bm = np.asarray(block_mask).astype(bool)
        ok &= bm[i // BLOCK, j // BLOCK]
    return ok


def dropout_threshold(p):
    """Integer threshold t for keep-iff-u16 >= t, from the float32 value of p."""
    p32 = float(np.float32(p))
    if not (0.0 <= p32 < 1.0):
        raise ValueError("dropout probability must lie in [0, 1)")
    return min(int(math.floor(p32 * 65536.0)), 65535)


def dropout_scale(p):
    """1 / keep probability = 2^16 / (2^16 - t): kept values are divided by it."""
    t = dropout_threshold(p)
    return 65536.0 / (65536.0 - t)


def dropout_keep(seed, p, b, h, rows, n, key0=0):
    """Keep bits Z[i, j] (bool) for query rows ``rows`` and keys key0..key0+n-1
    (rows and keys are positions in the whole sequence: the bits are keyed by
    them, whatever slice of the problem a caller evaluates)."""
    t = dropout_threshold(p)
    if t == 0:
        return np.ones((len(rows), n), dtype=bool)
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    k0, k1 = seed & 0xFFFFFFFF, seed >> 32
    rows = np.asarray(rows, dtype=np.uint64)[:, None]
    g_first = key0 // 8
    g_last = (key0 + n + 7) // 8  # one past the last block
    groups = np.arange(g_first, g_last, dtype=np.uint64)[None, :]
    words = philox4x32_10(groups, rows, np.uint64(h), np.uint64(b), k0, k1)
    # key 8 g + 2 m + s takes half s of word m of block g
    halves = []
    for w in words:
        halves.append(w & np.uint32(0xFFFF))
        halves.append(w >> np.uint32(16))
    u = np.stack(halves, axis=-1).reshape(len(rows), -1)
    start = key0 - 8 * g_first
    return u[:, start:start + n] >= np.uint32(t)


# ----------------------------------------------------------------------------
# the softmax step
# ----------------------------------------------------------------------------

def safe_softmax(s, valid):
    """Row-wise softmax over the valid entries of s, max-subtracted.

    Returns (P, lse, m, l).  Rows without a valid entry: P = 0, lse = -inf.
    """
    s = np.asarray(s, dtype=np.float64)
    masked = np.where(valid, s, -np.inf)
    m = masked.max(axis=1)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.where(valid, np.exp(masked - m_safe[:, None]), 0.0)
    l = e.sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        p = np.where(l[:, None] > 0, e / np.where(l > 0, l, 1.0)[:, None], 0.0)
        lse = np.where(l > 0, m_safe + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return p, lse, m, l


# ----------------------------------------------------------------------------
# forward
# ----------------------------------------------------------------------------

def _head_forward(q, k, v, scale, rows, causal, kv_len, block_mask, keep, rscale):
    s = scale * (q[rows] @ k.T)
    valid = valid_mask(k.shape[0], rows, causal, kv_len, block_mask, n_q=q.shape[0])
    p, lse, _, _ = safe_softmax(s, valid)
    pd = p if keep is None else p * keep * rscale
    return pd @ v, lse


def attention_forward(q, k, v, scale, causal=False, seqlens=None, dropout_p=0.0,
                      seed=0, block_mask=None, heads=None, rows=None, slab=256):
    """O and LSE of standard attention.

    q: float64 [B, H, N_q, d]; k, v: [B, H, N_k, d] (N_k may differ from N_q).
    Returns (O [B,H,R,d], LSE [B,H,R]) where R indexes ``rows`` (default all
    N_q rows).  ``heads`` optionally restricts the
    computation to a list of (b, h) pairs (other entries are left NaN).  Rows
    are processed in slabs of ``slab`` rows only to bound memory: every row is
    computed independently, so the slab size does not change any value.
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, H, N, d = q.shape
    Nk = k.shape[2]
    rows = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.full((B, H, rows.size, d), np.nan)
    lse = np.full((B, H, rows.size), np.nan)
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    p32 = float(np.float32(dropout_p))
    rscale = dropout_scale(p32)
    for b, h in pairs:
        kv_len = None if seqlens is None else int(seqlens[b])
        for r0 in range(0, rows.size, slab):
            rr = rows[r0:r0 + slab]
            keep = None
            if p32 > 0:
                keep = dropout_keep(seed, p32, b, h, rr, Nk)
            o, l = _head_forward(q[b, h], k[b, h], v[b, h], scale, rr, causal,
                                 kv_len, block_mask, keep, rscale)
            out[b, h, r0:r0 + rr.size] = o
            lse[b, h, r0:r0 + rr.size] = l
    return out, lse


# ----------------------------------------------------------------------------
# backward
# ----------------------------------------------------------------------------

def head_backward(q, k, v, dout, scale, causal=False, kv_len=None, block_mask=None,
                  keep=None, dropout_p=0.0):
    """dQ, dK, dV of one (b, h) by the chain rule through S, P, dropout, PV.

    The recomputation of the pages (rebuild P in the backward from saved
    statistics, suanlizi.com summary "重计算" and researchpapers.dev
    "分块与重计算") gives the same numbers as keeping P, which is what a
    standard implementation does; the oracle simply recomputes S and P here.
    """
    n = k.shape[0]
    rows = np.arange(q.shape[0])
    s = scale * (q @ k.T)
    valid = valid_mask(n, rows, causal, kv_len, block_mask, n_q=q.shape[0])
    p, _, _, _ = safe_softmax(s, valid)
    p32 = float(np.float32(dropout_p))
    if keep is None or p32 == 0:
        z = np.ones_like(p)
        rscale = 1.0
    else:
        z = keep.astype(np.float64)
        rscale = dropout_scale(p32)
    pd = p * z * rscale                 # dropped, rescaled P that multiplies V
    dv = pd.T @ dout                    # O = Pd V  ->  dV = Pd^T dO
    dpd = dout @ v.T                    # gradient w.r.t. Pd
    dp = dpd * z * rscale               # gradient w.r.t. P through the dropout
    dsum = (p * dp).sum(axis=1)         # softmax Jacobian term: sum_j P_ij dP_ij
    ds = p * (dp - dsum[:, None])       # gradient w.r.t. S
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv, dsum


def attention_backward(q, k, v, dout, scale, causal=False, seqlens=None,
                       dropout_p=0.0, seed=0, block_mask=None, heads=None):
    """dQ [B,H,N_q,d], dK, dV [B,H,N_k,d] (float64) for every (b, h) in
    ``heads`` (default all)."""
    q, k, v, dout = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dout))
    B, H, N, d = q.shape
    Nk = k.shape[2]
    dq = np.full_like(q, np.nan)
    dk = np.full_like(k, np.nan)
    dv = np.full_like(v, np.nan)
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    p32 = float(np.float32(dropout_p))
    for b, h in pairs:
        kv_len = None if seqlens is None else int(seqlens[b])
        keep = dropout_keep(seed, p32, b, h, np.arange(N), Nk) if p32 > 0 else None
        g = head_backward(q[b, h], k[b, h], v[b, h], dout[b, h], scale, causal,
                          kv_len, block_mask, keep, p32)
        dq[b, h], dk[b, h], dv[b, h] = g[0], g[1], g[2]
    return dq, dk, dv



# ----------------------------------------------------------------------------
# sampled backward, for checking full-size runs output by output
# ----------------------------------------------------------------------------

def _row_terms(q, k, v, dout, scale, rows, causal, kv_len, block_mask, keep, dropout_p):
    """P, the dropped P, and dS of the given query rows (each row needs only its
    own row of S, of dP = dO V^T and its own D_i)."""
    n = k.shape[0]
    s = scale * (q[rows] @ k.T)
    valid = valid_mask(n, rows, causal, kv_len, block_mask, n_q=q.shape[0])
    p, _, _, _ = safe_softmax(s, valid)
    p32 = float(np.float32(dropout_p))
    if keep is None or p32 == 0:
        z, rscale = 1.0, 1.0
    else:
        z, rscale = keep.astype(np.float64), dropout_scale(p32)
    pd = p * z * rscale
    dp = (dout[rows] @ v.T) * z * rscale
    dsum = (p * dp).sum(axis=1)
    ds = p * (dp - dsum[:, None])
    return pd, ds


def head_forward_rows(q, k, v, scale, rows, causal=False, kv_len=None, block_mask=None,
                      dropout_p=0.0, seed=0, b=0, h=0, row0=0, key0=0):
    """O and LSE of the given query rows of one (b, h) (q, k, v: [N, d]).
    row0 / key0: sequence positions of q's and k's first rows, where q, k, v
    are a slice of a larger problem (they place the dropout bits only)."""
    rows = np.asarray(rows, dtype=np.int64)
    p32 = float(np.float32(dropout_p))
    keep, rscale = None, 1.0
    if p32 > 0:
        keep = dropout_keep(seed, p32, b, h, rows + row0, k.shape[0], key0)
        rscale = dropout_scale(p32)
    return _head_forward(q, k, v, scale, rows, causal, kv_len, block_mask, keep, rscale)


def head_backward_rows(q, k, v, dout, scale, rows, causal=False, kv_len=None,
                       block_mask=None, dropout_p=0.0, seed=0, b=0, h=0, row0=0, key0=0):
    """dQ of the given query rows of one (b, h): scale * dS[rows] K (row0 /
    key0 as in head_forward_rows)."""
    rows = np.asarray(rows, dtype=np.int64)
    p32 = float(np.float32(dropout_p))
    keep = dropout_keep(seed, p32, b, h, rows + row0, k.shape[0], key0) if p32 > 0 else None
    _, ds = _row_terms(q, k, v, dout, scale, rows, causal, kv_len, block_mask, keep, p32)
    return scale * (ds @ k)


def head_backward_cols(q, k, v, dout, scale, cols, causal=False, kv_len=None,
                       block_mask=None, dropout_p=0.0, seed=0, b=0, h=0, slab=256,
                       rows=None, row0=0, key0=0):
    """dK and dV of the given key columns of one (b, h) (row0 / key0 as in
    head_forward_rows).

    Both are sums over query rows (dV_j = sum_i Pdrop_ij dO_i,
    dK_j = scale sum_i dS_ij Q_i); the rows are visited in slabs of ``slab``
    only to bound memory.  ``rows`` (default: all) limits the sum to a subset
    of query rows; it is only correct when every left-out row has P_ij = 0 for
    all the requested columns (e.g. rows whose blocks the block mask removes).
    """
    cols = np.asarray(cols, dtype=np.int64)
    n, d = k.shape
    p32 = float(np.float32(dropout_p))
    dk = np.zeros((cols.size, d))
    dv = np.zeros((cols.size, d))
    all_rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    for r0 in range(0, all_rows.size, slab):
        rows = all_rows[r0:r0 + slab]
        keep = dropout_keep(seed, p32, b, h, rows + row0, n, key0) if p32 > 0 else None
        pd, ds = _row_terms(q, k, v, dout, scale, rows, causal, kv_len, block_mask, keep, p32)
        dv += pd[:, cols].T @ dout[rows]
        dk += scale * (ds[:, cols].T @ q[rows])
    return dk, dv


# ----------------------------------------------------------------------------
# combining partial results over disjoint key sets
# ----------------------------------------------------------------------------

def merge_partials(o_a, lse_a, o_b, lse_b):
    """(O, LSE) over the union of two disjoint key sets from the results over
    each set alone: LSE = ln(e^LSE_a + e^LSE_b), O = e^(LSE_a - LSE) O_a +
    e^(LSE_b - LSE) O_b.  This is the definition of the softmax over a union
    (the normaliser is the sum of the parts' normalisers), the rule the
    pages' tiling applies between key blocks (suanlizi.com summary,
    分块计算（Tiling）).  Empty parts have LSE = -inf and add nothing."""
    o_a, o_b = np.asarray(o_a, dtype=np.float64), np.asarray(o_b, dtype=np.float64)
    lse_a, lse_b = np.asarray(lse_a, dtype=np.float64), np.asarray(lse_b, dtype=np.float64)
    m = np.maximum(lse_a, lse_b)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    ea = np.where(np.isneginf(lse_a), 0.0, np.exp(lse_a - m_safe))
    eb = np.where(np.isneginf(lse_b), 0.0, np.exp(lse_b - m_safe))
    s = ea + eb
    with np.errstate(divide="ignore", invalid="ignore"):
        lse = np.where(s > 0, m_safe + np.log(np.where(s > 0, s, 1.0)), -np.inf)
        wa = np.where(s > 0, ea / np.where(s > 0, s, 1.0), 0.0)
        wb = np.where(s > 0, eb / np.where(s > 0, s, 1.0), 0.0)
    return wa[..., None] * o_a + wb[..., None] * o_b, lse


def head_backward_block(q, k, v, dout, lse, delta, scale, causal=False, n_q=None, n_k=None,
                        q0=0, k0=0, dropout_p=0.0, seed=0, b=0, h=0):
    """The part of one head's backward that comes from one block of keys,
    given the softmax statistics of the full row (its LSE and
    D_i = sum_c dO_ic O_ic over all keys): with P = exp(scale Q K_blk^T - LSE),
    dP = dO V_blk^T and dS = P (dP - D),

        dQ_part = scale dS K_blk,  dK_blk = scale dS^T Q,  dV_blk = P^T dO.

    Summed over disjoint key blocks this is the full backward (the recomputation
    of the pages needs only LSE and D per row: suanlizi.com summary, 重计算).
    q, dout: [R, d] rows q0 .. of a sequence of n_q queries; k, v: [C, d] keys
    k0 .. of n_k keys; causal (bottom-right): key j valid iff j <= i + n_k - n_q.
    Dropout (the inverted dropout of attention_forward, keep bits Z keyed by the
    rows' and keys' positions in the sequence, q0 + i and k0 + j, of (b, h)):
    dV_blk = (P Z / q)^T dO and dP = (dO V_blk^T) Z / q, q the keep
    probability, while dS = P (dP - D) keeps the undropped P."""
    q, k, v, dout = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dout))
    rows = q0 + np.arange(q.shape[0])[:, None]
    cols = k0 + np.arange(k.shape[0])[None, :]
    s = scale * (q @ k.T)
    valid = np.ones(s.shape, dtype=bool)
    if causal:
        valid = cols <= rows + ((n_k or 0) - (n_q or 0))
    lse = np.asarray(lse, dtype=np.float64)[:, None]
    with np.errstate(invalid="ignore"):
        p = np.where(valid & np.isfinite(lse), np.exp(s - np.where(np.isfinite(lse), lse, 0.0)),
                     0.0)
    p32 = float(np.float32(dropout_p))
    z, rscale = 1.0, 1.0
    if p32 > 0:
        z = dropout_keep(seed, p32, b, h, q0 + np.arange(q.shape[0]), k.shape[0], k0)
        z, rscale = z.astype(np.float64), dropout_scale(p32)
    dp = (dout @ v.T) * z * rscale
    ds = p * (dp - np.asarray(delta, dtype=np.float64)[:, None])
    return scale * (ds @ k), scale * (ds.T @ q), (p * z * rscale).T @ dout


# ----------------------------------------------------------------------------
# grouped K / V heads (an extension the pages do not treat)
# ----------------------------------------------------------------------------

def gqa_expand(x, group, axis=1):
    """K or V with H_kv heads on `axis`, each repeated for the `group` query
    heads that share it: query head h reads K / V head h // group."""
    return np.repeat(np.asarray(x, dtype=np.float64), group, axis=axis)


def gqa_reduce(dx, group, axis=1):
    """The gradient of a K / V head shared by `group` query heads: the sum of
    the gradients of its copies (the chain rule through the repetition)."""
    dx = np.moveaxis(np.asarray(dx, dtype=np.float64), axis, 0)
    dx = dx.reshape((dx.shape[0] // group, group) + dx.shape[1:]).sum(axis=1)
    return np.moveaxis(dx, 0, axis)


def attention_forward_gqa(q, k, v, scale, causal=False, seqlens=None, dropout_p=0.0, seed=0,
                          block_mask=None):
    """O, LSE when k, v ([B, H_kv, N, d]) have fewer heads than q ([B, H, N, d]):
    standard attention against the K / V head of each query head's group.
    Dropout keeps its (b, h, i, j) keying with h the query head."""
    group = q.shape[1] // k.shape[1]
    return attention_forward(q, gqa_expand(k, group), gqa_expand(v, group), scale, causal,
                             seqlens, dropout_p, seed, block_mask)


def attention_backward_gqa(q, k, v, dout, scale, causal=False, seqlens=None, dropout_p=0.0,
                           seed=0, block_mask=None):
    """dQ [B, H, N, d] and dK, dV [B, H_kv, N, d] of attention_forward_gqa."""
    group = q.shape[1] // k.shape[1]
    dq, dk, dv = attention_backward(q, gqa_expand(k, group), gqa_expand(v, group), dout, scale,
                                    causal, seqlens, dropout_p, seed, block_mask)
    return dq, gqa_reduce(dk, group), gqa_reduce(dv, group)
