// Internal interface between the C ABI (fa_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "philox.cuh"

namespace fa {

// Grid order of the forward and backward CTAs.  Tile-major (all heads'
// heaviest tiles first, a longest-processing-time order) whenever the tiles
// differ in cost, i.e. under a causal mask, or when every head's K/V fits in
// L2 anyway; otherwise (equal-cost tiles, K/V beyond L2) head-major, so that
// the CTAs resident at one time share few heads and each head's K/V stays in
// L2.  (Measured on B200: causal 16K d=128 forward 983 -> 1066 TFLOP/s with
// the tile-major order; the 64K block-sparse backward 4517 -> 3702 without
// head-major locality.)
// The tile index then is the grid's y extent, which must stay within 65535.
inline bool tiles_major_order(int B, int H, int N, int d, bool causal) {
  const double kv_bytes = 4.0 * B * H * static_cast<double>(N) * d;  // K and V, bf16
  const bool tiles_fit_y = (N + 127) / 128 <= 65535;
  return tiles_fit_y && (causal || kv_bytes <= 48.0 * 1024 * 1024);
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
  int tiles_major;            // grid is (B*H, tiles) instead of (tiles, B*H)
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
  int tiles_major;            // grid is (B*H, tiles) instead of (tiles, B*H)
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
