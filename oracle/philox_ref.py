"""Philox counter-based generator, written from its published definition.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module:
it exists so that tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` can check the CUDA kernels against an independent restatement.

Source of the definition: J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw,
"Parallel Random Numbers: As Easy as 1, 2, 3", SC'11, section "Philox".
The attention pages only say that dropout is fused into the kernel
(suanlizi.com FlashAttention summary, description of Figure 1 right: the fused
kernel replaces separate matmul / dropout / softmax / mask steps); the choice of
Philox4x32-10 as the in-kernel dropout generator is the stated design of this
library, not something the pages fix.

Philox-N x W with R rounds (N = 4 words here):
  * state: a counter of 4 words of W bits and a key of 2 words of W bits;
  * one round multiplies word 0 and word 2 by two fixed odd multipliers, takes the
    high and low halves of each 2W-bit product, and permutes / xors them with the
    two untouched words and the key;
  * between rounds the key is advanced by two Weyl constants (the fractional
    parts of the golden ratio and of sqrt(3), scaled to W bits).

The round function is written once, generically in W, so that the 64-bit
instance can be pinned against numpy's independent ``numpy.random.Philox``
(Philox4x64-10) while the 32-bit instance is what dropout uses.
"""

from __future__ import annotations

import numpy as np

# Multipliers published in the Philox paper (table of Philox parameters).
PHILOX_M = {
    32: (0xD2511F53, 0xCD9E8D57),
    64: (0xD2E7470EE14C6C93, 0xCA5A826395121157),
}


def weyl_constants(width: int) -> tuple[int, int]:
    """Key increments: floor(2^w * (phi - 1)) and floor(2^w * (sqrt(3) - 1)).

    Computed from their mathematical definition with exact integer square roots,
    so no constant is typed in by hand.
    """
    from math import isqrt

    scale = 1 << width
    # phi - 1 = (sqrt(5) - 1) / 2  ->  floor(scale * (sqrt(5) - 1) / 2)
    s5 = isqrt(5 * scale * scale)           # floor(sqrt(5) * scale)
    w0 = (s5 - scale) // 2
    s3 = isqrt(3 * scale * scale)           # floor(sqrt(3) * scale)
    w1 = s3 - scale
    return w0, w1


def philox_block(counter, key, width: int = 32, rounds: int = 10):
    """One Philox4xW-R block on Python integers.

    counter: 4 ints (each < 2^width), key: 2 ints.  Returns the 4 output words.
    Slow, scalar, obviously written: used for pins and tiny cases.
    """
    mask = (1 << width) - 1
    m0, m1 = PHILOX_M[width]
    w0, w1 = weyl_constants(width)
    c0, c1, c2, c3 = (int(x) & mask for x in counter)
    k0, k1 = (int(x) & mask for x in key)
    for r in range(rounds):
        if r > 0:
            k0 = (k0 + w0) & mask
            k1 = (k1 + w1) & mask
        p0 = m0 * c0
        p1 = m1 * c2
        hi0, lo0 = p0 >> width, p0 & mask
        hi1, lo1 = p1 >> width, p1 & mask
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Vectorised Philox4x32-10 over numpy arrays (broadcasting).

    All inputs are integer arrays holding 32-bit values; the arithmetic is done
    in uint64 so that every 32x32-bit product is exact.  Returns four uint32
    arrays.  Same steps as ``philox_block`` with width 32.
    """
    mask = np.uint64(0xFFFFFFFF)
    m0, m1 = (np.uint64(m) for m in PHILOX_M[32])
    w0, w1 = (np.uint64(w) for w in weyl_constants(32))
    shape = np.broadcast_shapes(*(np.shape(x) for x in (c0, c1, c2, c3, k0, k1)))
    c0, c1, c2, c3, k0, k1 = (
        np.broadcast_to(np.asarray(x, dtype=np.uint64) & mask, shape).copy()
        for x in (c0, c1, c2, c3, k0, k1)
    )
    for r in range(10):
        if r > 0:
            k0 = (k0 + w0) & mask
            k1 = (k1 + w1) & mask
        p0 = m0 * c0
        p1 = m1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & mask
        hi1, lo1 = p1 >> np.uint64(32), p1 & mask
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return tuple(x.astype(np.uint32) for x in (c0, c1, c2, c3))
