"""Standard (unfused) attention on the GPU, written with plain PyTorch ops.

This is the comparison system of the pages, not part of the library: the
"PyTorch" bars of Figure 1 (right) in the suanlizi.com FlashAttention summary,
where matmul, mask, softmax, dropout and matmul run as separate kernels and
each one reads its input from HBM and writes its output back (same page,
section 核心操作融合).  The N x N score matrix S and the probability matrix P
are materialised in device memory, so memory grows as N^2 per head, against
O(N) for the fused kernels (researchpapers.dev "FlashAttention 详解", section
关键结果).

It exists to be timed beside the fused kernels on the same B200 and the same
inputs (bench.py), and its result is checked against the float64 oracle in
the GPU tests, so the timing compares two programs that compute the same
thing.  Dropout here draws its bits from torch's own generator: it has the
cost of standard dropout but not the library's Philox bits, so dropout runs
are timed but not compared element by element.

Nothing in ``io_aware_exact_20_b200`` imports this module.
"""

from __future__ import annotations


def valid_pairs(N, causal, seqlens, block_mask, device):
    """Boolean mask broadcastable to [B, H, N, N] (True = the pair takes part),
    or None when every pair does.  Same mask semantics as the library: causal
    j <= i, keys j >= seqlens[b] removed, 128 x 128 blocks of the block mask."""
    import torch
    valid = None
    if causal:
        valid = torch.ones(N, N, dtype=torch.bool, device=device).tril_()
    if block_mask is not None:
        bm = torch.as_tensor(block_mask, device=device).bool()
        idx = torch.arange(N, device=device) // 128
        blk = bm[idx][:, idx]
        valid = blk if valid is None else valid & blk
    if valid is not None:
        valid = valid[None, None]
    if seqlens is not None:
        lens = torch.as_tensor(seqlens, device=device).long()
        keys = torch.arange(N, device=device)[None, :] < lens[:, None]   # [B, N]
        keys = keys[:, None, None, :]
        valid = keys if valid is None else valid & keys
    return valid


def attention(q, k, v, scale, valid=None, dropout_p=0.0):
    """O = dropout(softmax(mask(scale Q K^T))) V as separate ops (autograd-able)."""
    import torch
    s = torch.matmul(q, k.transpose(-1, -2)) * scale
    if valid is not None:
        s = s.masked_fill(~valid, float("-inf"))
    p = torch.softmax(s, dim=-1)
    if dropout_p > 0:
        p = torch.nn.functional.dropout(p, p=dropout_p, training=True)
    return torch.matmul(p, v)


class UnfusedStep:
    """One forward + backward of standard attention on resident tensors."""

    def __init__(self, q, k, v, do, scale, causal=False, seqlens=None, dropout_p=0.0,
                 block_mask=None):
        self.q = q.detach().clone().requires_grad_(True)
        self.k = k.detach().clone().requires_grad_(True)
        self.v = v.detach().clone().requires_grad_(True)
        self.do = do
        self.scale = scale
        self.dropout_p = dropout_p
        self.valid = valid_pairs(q.shape[2], causal, seqlens, block_mask, q.device)

    def __call__(self):
        for t in (self.q, self.k, self.v):
            t.grad = None
        o = attention(self.q, self.k, self.v, self.scale, self.valid, self.dropout_p)
        o.backward(self.do)
        return o.detach(), self.q.grad, self.k.grad, self.v.grad
