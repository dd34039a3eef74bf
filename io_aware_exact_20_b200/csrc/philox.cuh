// Philox4x32-10 counter-based generator on the device, written from its
// published definition (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers:
// As Easy as 1, 2, 3", SC'11): ten rounds, each multiplying words 0 and 2 by
// fixed odd multipliers, swapping high/low halves with the other two words
// and the key, the key advanced between rounds by the Weyl constants
// floor(2^32 (phi - 1)) and floor(2^32 (sqrt(3) - 1)).
//
// Dropout keep bit of (b, h, i, j): one block at counter (j >> 3, i, h, b) with
// key (seed lo, seed hi) serves eight keys; key j takes the 16-bit half (j & 1)
// (0 = low) of word ((j >> 1) & 3) and is kept iff that value >= threshold.
#pragma once

#include <cstdint>

namespace fa {

struct Philox4 {
  uint32_t w0, w1, w2, w3;
};

__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                                 uint32_t c3, uint32_t k0, uint32_t k1) {
  constexpr uint32_t kMul0 = 0xD2511F53u, kMul1 = 0xCD9E8D57u;
  constexpr uint32_t kWeyl0 = 0x9E3779B9u, kWeyl1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += kWeyl0;
      k1 += kWeyl1;
    }
    const uint32_t hi0 = __umulhi(kMul0, c0), lo0 = kMul0 * c0;
    const uint32_t hi1 = __umulhi(kMul1, c2), lo1 = kMul1 * c2;
    const uint32_t n0 = hi1 ^ c1 ^ k0;
    const uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return Philox4{c0, c1, c2, c3};
}

// Round keys (k0 + r W0, k1 + r W1) for r = 0..9, computed once on the host
// and read from the kernel parameters, so that each round is two 32x32->64
// multiplies and two three-input xors.
struct PhiloxRoundKeys {
  uint32_t k0[10];
  uint32_t k1[10];
};

__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                                 uint32_t c3, const PhiloxRoundKeys& rk) {
  constexpr uint32_t kMul0 = 0xD2511F53u, kMul1 = 0xCD9E8D57u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = static_cast<uint64_t>(c0) * kMul0;
    const uint64_t p1 = static_cast<uint64_t>(c2) * kMul1;
    const uint32_t hi0 = static_cast<uint32_t>(p0 >> 32), lo0 = static_cast<uint32_t>(p0);
    const uint32_t hi1 = static_cast<uint32_t>(p1 >> 32), lo1 = static_cast<uint32_t>(p1);
    const uint32_t n0 = hi1 ^ c1 ^ rk.k0[r];
    const uint32_t n2 = hi0 ^ c3 ^ rk.k1[r];
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return Philox4{c0, c1, c2, c3};
}

// The eight keep bits of one block: bit k for key 8 g + k.
__device__ __forceinline__ uint32_t keep_byte(const Philox4& r, uint32_t thr) {
  return ((r.w0 & 0xFFFFu) >= thr ? 1u : 0u) | ((r.w0 >> 16) >= thr ? 2u : 0u) |
         ((r.w1 & 0xFFFFu) >= thr ? 4u : 0u) | ((r.w1 >> 16) >= thr ? 8u : 0u) |
         ((r.w2 & 0xFFFFu) >= thr ? 16u : 0u) | ((r.w2 >> 16) >= thr ? 32u : 0u) |
         ((r.w3 & 0xFFFFu) >= thr ? 64u : 0u) | ((r.w3 >> 16) >= thr ? 128u : 0u);
}

// Host-side round keys for a 64-bit seed.
inline PhiloxRoundKeys philox_round_keys(uint64_t seed) {
  PhiloxRoundKeys rk;
  uint32_t k0 = static_cast<uint32_t>(seed & 0xFFFFFFFFull), k1 = static_cast<uint32_t>(seed >> 32);
  for (int r = 0; r < 10; ++r) {
    rk.k0[r] = k0;
    rk.k1[r] = k1;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return rk;
}

}  // namespace fa
