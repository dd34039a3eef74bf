"""The QKV projection in front of attention, in float64 (the oracle of the
fused projection kernel).

TEST INFRASTRUCTURE ONLY (same rules as ``attention_ref``).

The pages' future-work section asks for the IO-aware treatment of the other
layers of the model, each of which reads and writes HBM (suanlizi.com
FlashAttention summary, section IO-感知优化的普遍性 / 子解法2).  The layer
that feeds attention is the projection of the token activations X into
queries, keys and values.  The pages do not define it; the plain reading is
the usual transformer one, with the three weight matrices stacked row-wise
into one [3 H d, D_model] matrix as a single linear layer stores them:

    Y = X W^T + bias,                        X: [T, D_model], T = B N tokens
    column c of Y = which * H d + h d + e,   which 0 = Q, 1 = K, 2 = V
    token t = b N + n,

so Q[b, h, n, e] = Y[b N + n, h d + e] (K, V likewise with offsets H d and
2 H d), each written as [B, H, N, d], the layout the attention kernels read.
"""

from __future__ import annotations

import numpy as np


def qkv_projection(x, w, bias, batch, heads, head_dim):
    """Q, K, V [B, H, N, d] (float64) from x [T, Dm], w [3 H d, Dm], bias [3 H d]
    or None; T must be batch * N."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    T = x.shape[0]
    H, d = heads, head_dim
    if w.shape[0] != 3 * H * d or w.shape[1] != x.shape[1] or T % batch:
        raise ValueError("shapes do not match")
    n = T // batch
    y = x @ w.T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    y = y.reshape(batch, n, 3, H, d)                 # [b, n, which, h, e]
    q, k, v = (y[:, :, i].transpose(0, 2, 1, 3) for i in range(3))  # [b, h, n, e]
    return q.copy(), k.copy(), v.copy()
