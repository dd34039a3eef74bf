"""Standard attention over packed variable-length batches, in float64.

TEST INFRASTRUCTURE ONLY (same rules as ``attention_ref``: imported only by
``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``).

The pages' BERT-large workload is a batch of sequences of different lengths
(researchpapers.dev "FlashAttention 详解", section 关键结果: BERT-large,
sequence length 512).  Stored packed, sequence b occupies the rows
cu[b] .. cu[b+1]-1 of a [T, H, d] tensor (no padding rows), and attention is
the standard attention of each sequence on its own: nothing crosses from one
sequence to another.  Per sequence b and head h this module calls the padded
oracle (``attention_ref``) on that sequence's rows, so every reading there
applies unchanged, with these positions:

  * i and j are positions inside sequence b (0-based), for the causal mask,
    the block mask and the dropout counter (j >> 3, i, h, b);
  * N_q = cu_q[b+1] - cu_q[b] and N_k = cu_k[b+1] - cu_k[b]; the causal mask
    is bottom-right aligned (query i sees key j iff j <= i + N_k - N_q);
  * an optional key length seqlens_k[b] further removes keys j >= seqlens_k[b]
    without moving the causal alignment;
  * block_mask is indexed by (i // 128, j // 128) inside the sequence.

Layouts: Q, O, dO, dQ [T_q, H, d]; K, V, dK, dV [T_k, H, d]; LSE [H, T_q].
"""

from __future__ import annotations

import numpy as np

from .attention_ref import _head_forward, dropout_keep, dropout_scale, head_backward


def _sequences(cu_q, cu_k):
    cu_q = np.asarray(cu_q, dtype=np.int64)
    cu_k = np.asarray(cu_k, dtype=np.int64)
    if cu_q.shape != cu_k.shape or cu_q.ndim != 1 or cu_q.size < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must be int arrays of B + 1 offsets")
    if (np.diff(cu_q) < 0).any() or (np.diff(cu_k) < 0).any() or cu_q[0] != 0 or cu_k[0] != 0:
        raise ValueError("cumulative lengths must start at 0 and not decrease")
    return [(int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1]))
            for b in range(cu_q.size - 1)]


def attention_forward_varlen(q, k, v, cu_q, cu_k, scale, causal=False, seqlens_k=None,
                             dropout_p=0.0, seed=0, block_mask=None):
    """O [T_q, H, d] and LSE [H, T_q] of standard attention per packed sequence."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    Tq, H, d = q.shape
    out = np.zeros((Tq, H, d))
    lse = np.full((H, Tq), -np.inf)
    p32 = float(np.float32(dropout_p))
    rscale = dropout_scale(p32)
    for b, (q0, q1, k0, k1) in enumerate(_sequences(cu_q, cu_k)):
        nq, nk = q1 - q0, k1 - k0
        if nq == 0 or nk == 0:  # no query, or no key: O = 0 and LSE = -inf
            continue
        kv_len = None if seqlens_k is None else min(max(int(seqlens_k[b]), 0), nk)
        rows = np.arange(nq)
        for h in range(H):
            keep = dropout_keep(seed, p32, b, h, rows, nk) if p32 > 0 else None
            o, l = _head_forward(q[q0:q1, h], k[k0:k1, h], v[k0:k1, h], scale, rows, causal,
                                 kv_len, block_mask, keep, rscale)
            out[q0:q1, h] = o
            lse[h, q0:q1] = l
    return out, lse


def attention_backward_varlen(q, k, v, dout, cu_q, cu_k, scale, causal=False, seqlens_k=None,
                              dropout_p=0.0, seed=0, block_mask=None):
    """dQ [T_q, H, d], dK, dV [T_k, H, d] of standard attention per packed sequence."""
    q, k, v, dout = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dout))
    Tq, H, d = q.shape
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    p32 = float(np.float32(dropout_p))
    for b, (q0, q1, k0, k1) in enumerate(_sequences(cu_q, cu_k)):
        nq, nk = q1 - q0, k1 - k0
        if nq == 0 or nk == 0:
            continue
        kv_len = None if seqlens_k is None else min(max(int(seqlens_k[b]), 0), nk)
        for h in range(H):
            keep = dropout_keep(seed, p32, b, h, np.arange(nq), nk) if p32 > 0 else None
            g = head_backward(q[q0:q1, h], k[k0:k1, h], v[k0:k1, h], dout[q0:q1, h], scale,
                              causal, kv_len, block_mask, keep, p32)
            dq[q0:q1, h], dk[k0:k1, h], dv[k0:k1, h] = g[0], g[1], g[2]
    return dq, dk, dv
