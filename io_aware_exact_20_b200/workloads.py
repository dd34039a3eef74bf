"""Seeded synthetic inputs shaped like the attention workloads on the pages.

This module holds no attention arithmetic: only random draws.  Both the CUDA
path's tests / benchmark and the float64 oracle receive the very same arrays
from here.  The pages benchmark GPT-2 (sequence 1K), BERT-large (sequence 512)
and long-sequence / block-sparse tasks (Path-X 16K, Path-256 64K); no dataset
is used anywhere: only the shapes are taken, and the values are drawn as below.

Recipe (shared by every workload):
  * Q, K, V, dO: float32 standard normal from ``numpy.random.default_rng(seed)``
    drawn in that order, each of shape [B, H, N, d], then rounded to bfloat16
    (round to nearest even, via torch);
  * key-padding lengths: integers uniform in [lo, hi] inclusive, one per batch
    entry, from ``default_rng(seed_len)``;
  * block mask: uint8 [nb, nb], nb = ceil(N / 128); the diagonal blocks are 1
    and every other block is 1 with probability ``density``, decided by
    ``default_rng(seed_mask).random((nb, nb)) < density``;
  * dropout seed: a 64-bit integer passed to the kernel as is.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool = False
    dropout_p: float = 0.0
    seqlen_range: tuple | None = None      # (lo, hi) inclusive, key padding
    block_density: float | None = None     # block-sparse mask density
    data_seed: int = 0
    dropout_seed: int = 0
    len_seed: int = 0
    mask_seed: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


def _wl(k, name, B, H, N, d, **kw):
    return Workload(name=name, B=B, H=H, N=N, d=d, data_seed=1000 + k,
                    dropout_seed=0x5EED0000 + k, len_seed=2000 + k,
                    mask_seed=3000 + k, **kw)


# The five workloads: tiny exact case, GPT-2-small-shaped causal with dropout,
# BERT-large-shaped key-padded with dropout, long causal sequence (d 64, 128
# and 256), and the 64K block-sparse case.
WORKLOADS = {
    "tiny": _wl(1, "tiny", 1, 2, 128, 64),
    "gpt2": _wl(2, "gpt2", 8, 12, 1024, 64, causal=True, dropout_p=0.1),
    "bert": _wl(3, "bert", 16, 16, 512, 64, dropout_p=0.1, seqlen_range=(256, 512)),
    "long64": _wl(4, "long64", 1, 16, 16384, 64, causal=True),
    "long128": _wl(4, "long128", 1, 16, 16384, 128, causal=True),
    "long256": _wl(4, "long256", 1, 16, 16384, 256, causal=True),
    "sparse": _wl(5, "sparse", 1, 8, 65536, 64, block_density=1.0 / 8.0),
}


def make_qkvdo(B, H, N, d, seed):
    """Q, K, V, dO as bfloat16 torch CPU tensors [B, H, N, d]."""
    import torch

    rng = np.random.default_rng(seed)
    out = []
    for _ in range(4):
        x = rng.standard_normal((B, H, N, d), dtype=np.float32)
        out.append(torch.from_numpy(x).to(torch.bfloat16))
    return tuple(out)


def make_seqlens(B, lo, hi, seed):
    """Per-batch valid key lengths, uniform integers in [lo, hi]."""
    rng = np.random.default_rng(seed)
    return rng.integers(lo, hi + 1, size=B, dtype=np.int64).astype(np.int32)


def make_block_mask(N, density, seed, block=128):
    """Diagonal blocks plus seeded random blocks at the given density."""
    nb = (N + block - 1) // block
    rng = np.random.default_rng(seed)
    m = (rng.random((nb, nb)) < density).astype(np.uint8)
    np.fill_diagonal(m, 1)
    return m


def make_inputs(w: Workload, B=None):
    """Everything a workload needs, as host arrays / CPU tensors.

    ``B`` overrides the batch size (used to shard the batch across ranks).
    """
    B = w.B if B is None else B
    q, k, v, do = make_qkvdo(B, w.H, w.N, w.d, w.data_seed)
    seqlens = None
    if w.seqlen_range is not None:
        seqlens = make_seqlens(B, w.seqlen_range[0], w.seqlen_range[1], w.len_seed)
    block_mask = None
    if w.block_density is not None:
        block_mask = make_block_mask(w.N, w.block_density, w.mask_seed)
    return dict(q=q, k=k, v=v, do=do, seqlens=seqlens, block_mask=block_mask,
                scale=w.scale, causal=w.causal, dropout_p=w.dropout_p,
                seed=w.dropout_seed)


def attention_flops(B, H, N, d, causal=False):
    """Nominal FLOPs (forward, backward): 4 B H N^2 d and 2.5 times that,
    both halved under a causal mask."""
    f = 4.0 * B * H * N * N * d
    if causal:
        f *= 0.5
    return f, 2.5 * f
