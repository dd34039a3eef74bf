// Internal interface between the C ABI (fa_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "philox.cuh"

namespace fa {

// Launches `kern` on `stream` with programmatic stream serialization: it may
// start launching while the previous kernel of the stream finishes its last
// wave (every kernel of the library waits for its predecessor with
// griddepcontrol.wait before touching global memory, see ptx.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_overlapped(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// Grid order of the forward and backward CTAs.  The 1-D grid walks groups of
// `group_heads` (b, h) heads one after the other and, inside a group, puts the
// tile index slowest: every head's heaviest tile first, a longest-processing-
// time order, which matters when a causal mask makes the tiles differ in
// cost.  The groups bound the bytes that the resident CTAs of a group share
// to about 48 MB, so that they stay in L2 and HBM traffic stays linear in N.
//   whole problem within 96 MB   -> one group (longest-first over all heads)
//   causal                       -> equal groups of at most 48 MB
//   no causal mask (equal tiles) -> one head per group (head-major)
// The forward's CTAs of one head share its K and V (bf16, 4 N d bytes); the
// backward's share the head's Q, dO (4 N d bytes), the fp32 dQ accumulators
// they all add into (4 N d) and the -LSE / -D rows (8 N).
// (Measured on B200, 16K causal d=128 forward: head-major 983 TFLOP/s,
// longest-first over all heads 1050-1066 with 1.4-3x the compulsory K/V reads.)
// Problems whose shared bytes fit in 96 MB (of the 126 MB L2) form one group;
// larger causal problems are cut into equal groups of at most 48 MB each (no
// short last group, which would run alone at the end of the grid).
inline int order_group_heads(int B, int H, double per_head_bytes, bool causal) {
  const int bh = B * H;
  const double mb = 1024.0 * 1024.0;
  if (per_head_bytes * bh <= 96.0 * mb) return bh;
  if (!causal) return 1;
  const double g = 48.0 * mb / per_head_bytes;
  if (g < 1.0) return 1;
  const int cap = g >= bh ? bh : static_cast<int>(g);
  const int groups = (bh + cap - 1) / cap;
  return (bh + groups - 1) / groups;
}
inline double fwd_head_bytes(int nk, int d) { return 4.0 * nk * d; }
inline double bwd_head_bytes(int nq, int d) { return 8.0 * nq * d + 8.0 * nq; }

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
enum : int { kStatusOk = 0, kStatusInternal = 3, kStatusTimeout = 4, kStatusBounds = 6 };

// Builds with FA_DEBUG_BOUNDS check every global-memory access the kernels
// make outside TMA (tensor maps clip by themselves) against the extent of its
// buffer: elements from the base pointer to one past the last element the call
// may touch, computed on the host from the call's sizes and strides.  An access
// out of range is skipped and kStatusBounds is recorded in the status word.
// Other builds compile the checks away (the macro drops its arguments).
#ifdef FA_DEBUG_BOUNDS
struct Extents {
  long long o, lse, dout, dq, dk, dv, mask, seqlens, kvacc;
};
__device__ __forceinline__ bool in_bounds(int* status, long long off, long long width,
                                          long long extent) {
  if (off >= 0 && width >= 0 && off + width <= extent) return true;
  if (status != nullptr) atomicExch(status, kStatusBounds);
  return false;
}
#define FA_IN_BOUNDS(status, off, width, extent) ::fa::in_bounds((status), (off), (width), (extent))
#else
#define FA_IN_BOUNDS(status, off, width, extent) true
#endif

// Element strides of a [batch, head, row, d] view (d is contiguous).
struct Strides {
  long long b, h, r;
};

// Where the rows of each batch entry live.  Padded layout (cu_q == null):
// every entry has nq query rows and nk key rows, at rows 0.. of its own
// batch slice.  Packed layout: entry b's queries are rows cu_q[b] ..
// cu_q[b+1]-1 of one [total_q] row range (keys likewise with cu_k), and nq,
// nk bound every sequence's length.
struct Rows {
  const int32_t* cu_q;
  const int32_t* cu_k;
  int nq, nk;
  int total_q, total_k;
#ifdef FA_DEBUG_BOUNDS
  long long n_cu;  // entries of cu_q and cu_k (B + 1)
  int* status;
#endif
};

// One batch entry resolved: first row and length of its queries and keys, and
// the batch coordinate of its tensors (0 when packed).  Offsets read from
// device memory are clamped so that no row falls outside the tensors.
struct Seq {
  int q0, lq, k0, lk, tb;
};

__device__ __forceinline__ Seq seq_of(const Rows& r, int b) {
  Seq s;
  if (r.cu_q == nullptr) {
    s.q0 = 0;
    s.lq = r.nq;
    s.k0 = 0;
    s.lk = r.nk;
    s.tb = b;
  } else {
    if (!FA_IN_BOUNDS(r.status, b, 2, r.n_cu)) return Seq{0, 0, 0, 0, 0};
    const int a0 = min(max(r.cu_q[b], 0), r.total_q);
    const int a1 = min(max(r.cu_q[b + 1], a0), r.total_q);
    const int c0 = min(max(r.cu_k[b], 0), r.total_k);
    const int c1 = min(max(r.cu_k[b + 1], c0), r.total_k);
    s.q0 = a0;
    s.lq = min(a1 - a0, r.nq);
    s.k0 = c0;
    s.lk = min(c1 - c0, r.nk);
    s.tb = 0;
  }
  return s;
}

struct FwdParams {
  void* o;                    // bf16, strides so
  Strides so;
  float* lse;                 // fp32 [B,H,nq] (padded) or [H,total_q] (packed)
  long long lse_sb, lse_sh;   // LSE element strides of a batch entry and a head
  const int32_t* seqlens;     // key lengths int32 [B] or null
  const uint8_t* block_mask;  // uint8 [nbq][nbk] or null
  int nbq, nbk;
  int* status;                // device status word
  Rows rows;
  int B, H, d_real;           // d_real <= the kernel's D: columns that exist
  float scale_log2;           // softmax_scale * log2(e)
  int causal;                 // bottom-right aligned: key j <= i + lk - lq
  int group_heads;            // grid order: heads per group (see order_group_heads)
  uint32_t drop_threshold;    // keep iff word >= threshold
  float drop_rscale;          // 1 / (1 - p)
  uint32_t seed_lo, seed_hi;
  PhiloxRoundKeys rk;         // round keys of the dropout generator
  uint32_t drop_row0;         // dropout counter: position of the call's row 0 ...
  uint32_t drop_kgrp0;        // ... and 8-key group of its key 0 in the keyed sequence
  uint64_t timeout_ns;
  int mask_bitmap;            // block masks: 1 = walk them through a shared-memory bitmask
  int group;                  // query heads per K / V head (1 = one K / V head each)
#ifdef FA_DEBUG_BOUNDS
  Extents ext;
#endif
};

struct BwdParams {
  const void* o;              // bf16 forward output
  const void* dout;           // bf16
  const float* lse;           // fp32, layout as in FwdParams
  long long lse_sb, lse_sh;
  void* dq;                   // bf16
  void* dk;                   // bf16
  void* dv;                   // bf16
  Strides so, sdo, sdq, sdk, sdv;
  // Workspace, three arrays of ws_rows rows each (row of (b, h, i) =
  // ws_row0(b, h) + i, every (b, h) owning its query rows rounded up to a
  // multiple of 128): -LSE * log2(e) (-inf where no key), -D_i, and D fp32
  // dQ accumulators per row (unscaled).
  float* ws_lse2;
  float* ws_delta;
  float* ws_dq;
  long long ws_rows;
  int Npad;                   // padded layout: rows per (b, h)
  long long Rtot;             // packed layout: rows per head
  const int32_t* seqlens;
  const uint8_t* block_mask;
  int nbq, nbk;
  int* status;
  Rows rows;
  int B, H, d_real;
  float scale;                // softmax_scale
  float scale_log2;           // softmax_scale * log2(e)
  int causal;
  int group_heads;            // grid order: heads per group (see order_group_heads)
  uint32_t drop_threshold;
  float drop_rscale;
  uint32_t seed_lo, seed_hi;
  PhiloxRoundKeys rk;
  uint32_t drop_row0, drop_kgrp0;  // as in FwdParams
  uint64_t timeout_ns;
  int mask_bitmap;            // as in FwdParams
  int group;                  // query heads per K / V head; the main kernel's units are
                              // (b, K / V head, key tile) and walk the group's query heads
  int split;                  // > 1: each unit splits into `split` parts, part p walking
                              // query heads [p, p + 1) * group / split of the group and
                              // writing its dK / dV to slice p of ws_dk / ws_dv
  int rows_tb;                // batch coordinates of the tensors (B padded, 1 packed)
  // fp32 dK / dV slices [split][rows_tb][H_kv][key rows][D] when split > 1
  float* ws_dk;
  float* ws_dv;
#ifdef FA_DEBUG_BOUNDS
  Extents ext;
#endif
};

// First workspace row of (b, h); a multiple of 128.  Packed sequences are
// spaced 256 rows apart from one another in addition to their offsets (rounded
// down to 128), which leaves every sequence room for its last, partial tile.
__host__ __device__ inline long long ws_row0(const BwdParams& p, int b, int h, int q0) {
  if (p.rows.cu_q == nullptr) return (static_cast<long long>(b) * p.H + h) * p.Npad;
  return static_cast<long long>(h) * p.Rtot + 128ll * (q0 / 128) + 256ll * b;
}

cudaError_t launch_fwd(int d, bool dropout, const CUtensorMap& tq, const CUtensorMap& tk,
                       const CUtensorMap& tv, const FwdParams& p, cudaStream_t stream);

// Backward in three launches: D / log2-LSE / zeroed dQ accumulators, the main
// kernel (dK, dV, dQ accumulators), and the dQ conversion.
cudaError_t launch_bwd_pre(int d, const BwdParams& p, cudaStream_t stream);
cudaError_t launch_bwd_main(int d, bool dropout, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, const CUtensorMap& tdo, const CUtensorMap& tdq,
                            const BwdParams& p, cudaStream_t stream);
cudaError_t launch_bwd_post(int d, const BwdParams& p, cudaStream_t stream);
// dK, dV from the fp32 accumulators of split units (BwdParams::split > 1)
cudaError_t launch_bwd_kv_post(int d, const BwdParams& p, cudaStream_t stream);

// Fused QKV projection (fa_proj.cu): x bf16 [B N, d_model], w bf16
// [3 H d, d_model], bias bf16 [3 H d] or null -> q, k, v bf16 [B, H, N, d].
cudaError_t launch_qkv_projection(const void* x, const void* w, const void* bias, void* q, void* k,
                                  void* v, int B, int N, int H, int d, int d_model, int* status,
                                  uint64_t timeout_ns, cudaStream_t stream);

cudaError_t launch_dropout_mask(uint8_t* keep, int B, int H, int N, uint32_t threshold,
                                uint32_t seed_lo, uint32_t seed_hi, cudaStream_t stream);

cudaError_t launch_wait_timeout_probe(int* status, uint64_t timeout_ns, cudaStream_t stream);

}  // namespace fa
