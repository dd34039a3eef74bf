// Internal interface between the C ABI (fa_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "philox.cuh"

namespace fa {

// Grid order of the forward and backward CTAs.  The 1-D grid walks groups of
// `group_heads` (b, h) heads one after the other and, inside a group, puts the
// tile index slowest: every head's heaviest tile first, a longest-processing-
// time order, which matters when a causal mask makes the tiles differ in
// cost.  The groups bound the K/V bytes that the resident CTAs read to about
// 48 MB, so that K and V stay in L2 and HBM traffic stays linear in N.
//   all heads' K/V within 48 MB  -> one group (longest-first over all heads)
//   causal                       -> groups of 48 MB of K/V
//   no causal mask (equal tiles) -> one head per group (head-major)
// (Measured on B200, 16K causal d=128 forward: head-major 983 TFLOP/s,
// longest-first over all heads 1050-1066 with 1.4-3x the compulsory K/V reads.)
inline int order_group_heads(int B, int H, int N, int d, bool causal) {
  const int bh = B * H;
  const double per_head = 4.0 * static_cast<double>(N) * d;  // K and V of one head, bf16
  const double budget = 48.0 * 1024 * 1024;
  if (per_head * bh <= budget) return bh;
  if (!causal) return 1;
  const double g = budget / per_head;
  return g < 1.0 ? 1 : (g >= bh ? bh : static_cast<int>(g));
}

// CTA u of a grid of bh_total x tiles work units -> (head, tile index).
__host__ __device__ inline void grid_unit(long long u, int bh_total, int tiles, int group_heads,
                                          int* bh, int* tile) {
  const long long per_group = static_cast<long long>(group_heads) * tiles;
  const long long grp = u / per_group;
  const int h0 = static_cast<int>(grp) * group_heads;
  const int gsz = bh_total - h0 < group_heads ? bh_total - h0 : group_heads;
  const long long r = u - grp * per_group;
  *tile = static_cast<int>(r / gsz);
  *bh = h0 + static_cast<int>(r % gsz);
}

// Device status codes written to the per-device status word.
enum : int { kStatusOk = 0, kStatusInternal = 3, kStatusTimeout = 4 };

struct FwdParams {
  void* o;                    // bf16 [B,H,N,d]
  float* lse;                 // fp32 [B,H,N]
  const int32_t* seqlens;     // int32 [B] or null
  const uint8_t* block_mask;  // uint8 [nblk][nblk] or null
  int* status;                // device status word
  int B, H, N, nblk;
  float scale_log2;           // softmax_scale * log2(e)
  int causal;
  int group_heads;            // grid order: heads per group (see order_group_heads)
  uint32_t drop_threshold;    // keep iff word >= threshold
  float drop_rscale;          // 1 / (1 - p)
  uint32_t seed_lo, seed_hi;
  PhiloxRoundKeys rk;         // round keys of the dropout generator
  uint64_t timeout_ns;
};

struct BwdParams {
  const void* o;              // bf16 [B,H,N,d]  (forward output)
  const void* dout;           // bf16 [B,H,N,d]
  const float* lse;           // fp32 [B,H,N]
  void* dq;                   // bf16 [B,H,N,d]
  void* dk;                   // bf16 [B,H,N,d]
  void* dv;                   // bf16 [B,H,N,d]
  float* ws_lse2;             // fp32 [B*H][Npad]  -LSE * log2(e), -inf where no key
  float* ws_delta;            // fp32 [B*H][Npad]  -sum_c dO_ic O_ic
  float* ws_dq;               // fp32 [B*H][Npad][d] dQ accumulators (unscaled)
  const int32_t* seqlens;
  const uint8_t* block_mask;
  int* status;
  int B, H, N, Npad, nblk;
  float scale;                // softmax_scale
  float scale_log2;           // softmax_scale * log2(e)
  int causal;
  int group_heads;            // grid order: heads per group (see order_group_heads)
  uint32_t drop_threshold;
  float drop_rscale;
  uint32_t seed_lo, seed_hi;
  PhiloxRoundKeys rk;
  uint64_t timeout_ns;
};

cudaError_t launch_fwd(int d, bool dropout, const CUtensorMap& tq, const CUtensorMap& tk,
                       const CUtensorMap& tv, const FwdParams& p, cudaStream_t stream);

// Backward in three launches: D / log2-LSE / zeroed dQ accumulators, the main
// kernel (dK, dV, dQ accumulators), and the dQ conversion.
cudaError_t launch_bwd_pre(int d, const BwdParams& p, cudaStream_t stream);
cudaError_t launch_bwd_main(int d, bool dropout, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, const CUtensorMap& tdo, const CUtensorMap& tdq,
                            const BwdParams& p, cudaStream_t stream);
cudaError_t launch_bwd_post(int d, const BwdParams& p, cudaStream_t stream);

cudaError_t launch_dropout_mask(uint8_t* keep, int B, int H, int N, uint32_t threshold,
                                uint32_t seed_lo, uint32_t seed_hi, cudaStream_t stream);

cudaError_t launch_wait_timeout_probe(int* status, uint64_t timeout_ns, cudaStream_t stream);

}  // namespace fa
