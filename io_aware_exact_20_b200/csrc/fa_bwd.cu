// Backward pass of exact attention on sm_100a.
//
// The probabilities are not stored by the forward pass: they are rebuilt here
// from the saved log-sum-exp (the recomputation of the pages: keep the softmax
// statistics, recompute the attention blocks in the backward).  With
// P = exp(S - LSE), dP = dO V^T (times the dropout keep / (1 - p)),
// D_i = sum_c dO_ic O_ic and dS = P * (dP - D):
//
//   dV = P_drop^T dO,   dK = scale dS^T Q,   dQ = scale dS K.
//
// Three kernels:
//   bwd_pre   -D_i, -LSE_i * log2(e) (-inf for rows without keys and
//             padding rows, so that their P is exactly 0), zeroed dQ
//             accumulators;
//   bwd_main  one CTA per (b, h, 128-key tile), looping over the query tiles
//             that tile meets; dK, dV stay in TMEM for the whole loop, dQ
//             partial products are added into fp32 accumulators;
//   bwd_post  dQ = bf16(scale * accumulator).
//
// bwd_main roles (512 threads):
//   warp 0        TMA producer: K, V once; per query tile Q, dO and the
//                 128-row slices of LSE*log2e and D into a ring
//   warp 1        TMEM allocator and single-thread MMA issuer
//   warps 4-11    two warpgroups, thread = key row; warpgroup w handles the
//                 query columns [64 w, 64 w + 64) in two phases per query
//                 tile: P from S^T (bf16 back to TMEM), then dS from dP^T
//                 (bf16 to swizzled shared memory)
//
// Per query tile the MMA warp issues dV as soon as P is in TMEM and the next
// tile's S^T right behind it, both while the dS phase runs; dK and dQ follow
// the dS phase and overlap the next tile's P phase.
//   warps 12-15   dQ warpgroup.  d = 64: TMEM -> the just-consumed Q / dO
//                 stage (128-byte-swizzled fp32 boxes of 32 columns x 128
//                 rows) -> TMA bulk reduce-add into the fp32 accumulators;
//                 the stage goes back to the producer once the reduce has
//                 read it.  d = 128: TMEM -> red.global.add of the transposed
//                 tile, one coalesced 128-byte line per warp instruction
//
// TMEM columns: S^T [0,128) with P packed into [64 w, 64 w + 32) per
// warpgroup; dP^T [128,256); dV [256, 256 + D); dK [256 + D, 256 + 2 D); the
// dQ tile in [384, 448) for d = 64; for d = 128 its transpose dQ^T (lane =
// feature, column = query) in the dP^T columns once dP^T has been consumed.
//
// d = 256 (and 192): the dK, dV accumulators of a key tile would fill TMEM on
// their own, so two CTAs share the tile, CTA h owning feature columns
// [128 h, 128 h + 128) of dK, dV and dQ; both compute the full S^T and dP^T.
// Each then has the d = 128 TMEM map (dV and dK halves of 128 columns, the dQ^T
// half in the dP^T columns) and the same roles; K and V stay resident, Q and
// dO pass through a ring of four 64-column panels that the producer fills in
// exactly the order the MMA warp takes them, and the LSE / D slices through a
// two-stage ring of their own that the P / dS warps hand back after their dS
// phase.
#include <cuda_bf16.h>

#include <type_traits>

#include "devctx.h"
#include "kernels.h"
#include "philox.cuh"
#include "ptx.cuh"

namespace fa {
namespace {

constexpr int kBwdThreads = 512;
constexpr float kLog2e = 1.44269504088896340736f;

template <int D>
struct BwdLayout {
  static constexpr int PANELS = D / 64;
  static constexpr uint32_t PANEL = 128u * 128u;
  static constexpr uint32_t TILE = PANEL * PANELS;
  // d = 256: two CTAs per key tile, each owning HD = 128 of the feature
  // columns of dK, dV and dQ (both recompute S^T and dP^T over all 256).
  // K and V stay resident; Q and dO pass through a ring of 64-column panels
  // in the order the MMAs consume them.
  static constexpr bool RING = (D == 256);
  static constexpr int HD = RING ? 128 : D;
  // Q / dO stages, or (RING) panel slots
  static constexpr int STAGES = RING ? 4 : (D == 64) ? 3 : 2;
  static constexpr int LD_STAGES = RING ? 2 : STAGES;
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = TILE;
  static constexpr uint32_t OFF_Q = 2 * TILE;  // RING: the panel slots
  static constexpr uint32_t OFF_DO = OFF_Q + (RING ? STAGES * PANEL : STAGES * TILE);
  static constexpr uint32_t OFF_DS = OFF_DO + (RING ? 0 : STAGES * TILE);  // [128 keys][128 queries] bf16
  static constexpr uint32_t OFF_LD = OFF_DS + 2 * PANEL;  // per stage: -lse2[128], -delta[128]
  static constexpr uint32_t OFF_BAR = OFF_LD + LD_STAGES * 1024;
  static constexpr int B_KV = 0;
  static constexpr int B_QFULL = 1;
  static constexpr int B_QEMPTY = B_QFULL + STAGES;
  static constexpr int B_SFULL = B_QEMPTY + STAGES;
  static constexpr int B_DPFULL = B_SFULL + 1;
  static constexpr int B_PFULL = B_DPFULL + 1;   // P of the tile is in TMEM
  static constexpr int B_DSFULL = B_PFULL + 1;   // dS of the tile is in shared memory
  static constexpr int B_DSEMPTY = B_DSFULL + 1;
  static constexpr int B_DQFULL = B_DSEMPTY + 1;
  static constexpr int B_DQEMPTY = B_DQFULL + 1;
  static constexpr int B_KVDONE = B_DQEMPTY + 1;
  static constexpr int B_STAGED = B_KVDONE + 1;   // dQ tile written to the staging boxes
  static constexpr int B_LDFULL = B_STAGED + 1;   // RING: the LSE / D slices of a query tile
  static constexpr int B_LDEMPTY = B_LDFULL + 2;
  static constexpr int NBAR = RING ? B_LDEMPTY + 2 : B_STAGED + 1;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
  // block masks at d = 64: bitmask of the query tiles this key tile meets
  // (up to 32 BIT_WORDS query tiles).  d = 128 keeps the direct walk: its
  // producer / MMA warps run at 72 registers, which the bitmask walk exceeds.
  static constexpr int BIT_WORDS = (D == 64) ? 1024 : 0;
  static constexpr uint32_t OFF_BITS = OFF_MISC + 16;
  static constexpr uint32_t SMEM = OFF_BITS + BIT_WORDS * 4;
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 256 + HD;
  // d = 64 leaves room for a dQ tile of its own; d = 128 and 256 reuse the
  // dP^T columns once dP^T has been consumed.
  static constexpr bool SEPARATE_DQ = (COL_DK + HD + HD <= 512);
  static constexpr uint32_t COL_DQ = SEPARATE_DQ ? COL_DK + HD : COL_DP;
  // d = 128 / 256: the dQ tile (its HD columns) is computed transposed
  // (dQ^T = K^T dS^T, TMEM lane = feature c, column = query) so that each
  // warp's reduction into the fp32 accumulators covers 32 consecutive floats
  // of one row: one 128-byte line.
  static constexpr bool DQ_T = (D == 128 || RING);
  // d = 64: the dQ tile is staged in the just-consumed Q / dO stage and added
  // into the accumulators by TMA bulk reduce-adds (the dQ warps then hand the
  // stage back to the producer).  d = 128 keeps the transposed tile and its
  // coalesced reductions: there a 64 KB stage of the two-deep Q / dO ring
  // held until the reduce has read it costs more than it saves.
  static constexpr bool TMA_REDUCE = !DQ_T;
  // d = 128 / 256: setmaxnreg moves registers from warpgroup 0 (producer,
  // MMA issuer) to the dQ warpgroup, which reads the whole transposed dQ tile
  // (128 values per thread) out of TMEM before it starts the reductions, so
  // that the TMEM columns it shares with the next tile's dP^T are free early.
  // 128 * (REGS_CTL + 2 * 128 + REGS_DQ) must equal 512 threads x 128.
  static constexpr bool SPLIT_REGS = DQ_T;
  static constexpr uint32_t REGS_CTL = 72;
  static constexpr uint32_t REGS_DQ = 184;
  static_assert(REGS_CTL + 2 * 128 + REGS_DQ == 4 * 128, "register split");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(COL_DK + HD <= 512, "TMEM budget");
  static_assert(!RING || BIT_WORDS == 0, "no room for the bitmask next to the ring");
};

// The key tile of this CTA and the query tiles that meet it.  Rows and keys
// are counted inside the CTA's sequence; qrow / krow are the tensor rows of the
// sequence's first query / key, tb its batch coordinate and ws0 its first
// workspace row.  Under the causal mask query i sees key j iff j <= i + off
// (bottom-right alignment, off = keys - queries of the sequence).
//
// Under a block mask the CTA first gathers the query tiles its key tile meets
// into a bitmask in shared memory (one pass over the mask column); the roles
// then find their next query tile with a word read and a find-first-set.
// Kernels launched without a block mask, with columns longer than the
// bitmask, or at d = 128 are built without it (kBits false) and test the
// mask's bytes directly.
// One step of a CTA's walk: query tile qb of the group's query head g,
// packed as g * 2^16 + qb (qb < 2^16 since N <= 2^23) by the general (GEN)
// instances; the others have one query head per K / V head and walk the query
// tile index itself.
using Tile = int;
template <bool GEN>
__device__ __forceinline__ int tile_g(Tile t) { return GEN ? t >> 16 : 0; }
template <bool GEN>
__device__ __forceinline__ int tile_qb(Tile t) { return GEN ? t & 0xFFFF : t; }

template <bool kBits>
struct BwdWork {
  int b, hk, bh, kb, kv_len, nqb, qb_begin, nbk, off, qrow, krow, tb, lk;  // hk: K / V head
  long long ws0;  // first workspace row of the first query head the CTA walks
  bool alive, causal;
  const uint8_t* bm;
  const uint32_t* bits;  // shared-memory bitmask over the query tiles, or null
#ifdef FA_DEBUG_BOUNDS
  int* status;
  long long ext_mask;
#endif

  __device__ __forceinline__ bool act(int qb) const {
    if (!alive) return false;
    if (bm != nullptr) {
      const long long mi = static_cast<long long>(qb) * nbk + kb;
      if (!FA_IN_BOUNDS(status, mi, 1, ext_mask) || bm[mi] == 0) return false;
    }
    return true;
  }
  __device__ __forceinline__ int next(int qb) const {
    if (kBits && bits != nullptr) {
      while (qb < nqb) {
        const uint32_t x = bits[qb >> 5] >> (qb & 31);
        if (x != 0u) return min(qb + __ffs(x) - 1, nqb);
        qb = (qb | 31) + 1;
      }
      return nqb;
    }
    while (qb < nqb && !act(qb)) ++qb;
    return qb;
  }
  // The walk.  GEN: over the G query heads of the group, the same query
  // tiles for each (the masks do not depend on the head), head after head;
  // done when tile_g(t) == G.  Otherwise: the query tiles, done at nqb.
  template <bool GEN>
  __device__ __forceinline__ Tile first(int G) const {
    const int qb = next(qb_begin);
    return GEN && qb >= nqb ? (G << 16) : qb;
  }
  template <bool GEN>
  __device__ __forceinline__ Tile step(Tile t) const {
    if constexpr (!GEN) {
      return next(t + 1);
    } else {
      const int qb = next(tile_qb<true>(t) + 1);
      return qb < nqb ? ((t & ~0xFFFF) | qb) : (((t & ~0xFFFF) + 0x10000) | next(qb_begin));
    }
  }
  template <bool GEN>
  __device__ __forceinline__ bool more(Tile t, int G) const {
    return GEN ? tile_g<true>(t) < G : t < nqb;
  }
  // query head of step t (base: the first query head the CTA walks), and the
  // workspace row of its query tile's first row (ws_hs: workspace rows from
  // one query head to the next)
  template <bool GEN>
  __device__ __forceinline__ int hq(Tile t, int base) const { return base + tile_g<GEN>(t); }
  template <bool GEN>
  __device__ __forceinline__ long long wsrow(Tile t, long long ws_hs) const {
    return ws0 + tile_g<GEN>(t) * ws_hs + 128ll * tile_qb<GEN>(t);
  }
};

// ---------------------------------------------------------------------------
// pre / post kernels
// ---------------------------------------------------------------------------

// Grid of the pre / post kernels: blockIdx.y = (b, h), blockIdx.x = a block
// of kRowsPerBlock<D> query rows, D / 8 threads per row (8 columns each).
template <int D>
constexpr int kRowsPerBlock = 256 / (D / 8);

template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const BwdParams p) {
  constexpr int G = D / 8;  // threads per row, 8 elements each
  griddep_wait();
  griddep_launch_dependents();
  const int bh = blockIdx.y;
  const int b = bh / p.H, h = bh % p.H;
  const Seq sq = seq_of(p.rows, b);
  const int i = blockIdx.x * kRowsPerBlock<D> + static_cast<int>(threadIdx.x) / G;
  const int part = static_cast<int>(threadIdx.x) % G;
  // rows up to the next multiple of 128 are written (padding rows included);
  // the bound is a multiple of the block's rows, so whole blocks leave
  if (blockIdx.x * kRowsPerBlock<D> >= (sq.lq + 127) / 128 * 128) return;
  float acc = 0.f;
  const long long r = sq.q0 + i;
  const long long o_off = sq.tb * p.so.b + h * p.so.h + r * p.so.r + part * 8;
  const long long do_off = sq.tb * p.sdo.b + h * p.sdo.h + r * p.sdo.r + part * 8;
  if (i < sq.lq && part * 8 < p.d_real && FA_IN_BOUNDS(p.status, o_off, 8, p.ext.o) &&
      FA_IN_BOUNDS(p.status, do_off, 8, p.ext.dout)) {
    const uint4 ov = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.o) + o_off);
    const uint4 gv = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.dout) + do_off);
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 a = __bfloat1622float2(o2[k]);
      const float2 c = __bfloat1622float2(g2[k]);
      acc = fmaf(a.x, c.x, acc);
      acc = fmaf(a.y, c.y, acc);
    }
  }
#pragma unroll
  for (int m = G / 2; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  const long long row = ws_row0(p, b, h, sq.q0) + i;
  if (part == 0 && FA_IN_BOUNDS(p.status, row, 1, p.ws_rows)) {
    p.ws_delta[row] = (i < sq.lq) ? -acc : 0.f;
    float nl2 = -INFINITY;
    const long long lse_off = sq.tb * p.lse_sb + h * p.lse_sh + sq.q0 + i;
    if (i < sq.lq && FA_IN_BOUNDS(p.status, lse_off, 1, p.ext.lse)) {
      const float l = p.lse[lse_off];
      if (l != -INFINITY) nl2 = -l * kLog2e;
    }
    p.ws_lse2[row] = nl2;
  }
  if (FA_IN_BOUNDS(p.status, row * D + part * 8, 8, p.ws_rows * D)) {
    float4* dq = reinterpret_cast<float4*>(p.ws_dq + row * D + part * 8);
    dq[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    dq[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

template <int D>
__global__ void __launch_bounds__(256) bwd_post_kernel(const BwdParams p) {
  constexpr int G = D / 8;
  griddep_wait();
  griddep_launch_dependents();
  const int bh = blockIdx.y;
  const int b = bh / p.H, h = bh % p.H;
  const Seq sq = seq_of(p.rows, b);
  const int i = blockIdx.x * kRowsPerBlock<D> + static_cast<int>(threadIdx.x) / G;
  const int part = static_cast<int>(threadIdx.x) % G;
  if (i >= sq.lq || part * 8 >= p.d_real) return;
  const long long acc_off = (ws_row0(p, b, h, sq.q0) + i) * D + part * 8;
  const long long dq_off = sq.tb * p.sdq.b + h * p.sdq.h + static_cast<long long>(sq.q0 + i) * p.sdq.r +
                           part * 8;
  if (!FA_IN_BOUNDS(p.status, acc_off, 8, p.ws_rows * D) ||
      !FA_IN_BOUNDS(p.status, dq_off, 8, p.ext.dq))
    return;
  const float4* src = reinterpret_cast<const float4*>(p.ws_dq + acc_off);
  const float4 a = src[0], c = src[1];
  const float s = p.scale;
  uint4 out;
  out.x = pack_bf16(a.x * s, a.y * s);
  out.y = pack_bf16(a.z * s, a.w * s);
  out.z = pack_bf16(c.x * s, c.y * s);
  out.w = pack_bf16(c.z * s, c.w * s);
  *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dq) + dq_off) = out;
}

// dK, dV = bf16(sum over the parts' fp32 slices) of split units (grouped K / V
// heads), the parts added in order: grid (blocks of kRowsPerBlock<D> key rows
// of the longest sequence) x (B * H_kv).  The slices hold scaled gradients.
template <int D>
__global__ void __launch_bounds__(256) bwd_kv_post_kernel(const BwdParams p) {
  constexpr int G = D / 8;
  griddep_wait();
  griddep_launch_dependents();
  const int n_kv = p.H / p.group;
  const int bh = blockIdx.y;
  const int b = bh / n_kv, hk = bh % n_kv;
  const Seq sq = seq_of(p.rows, b);
  const int j = blockIdx.x * kRowsPerBlock<D> + static_cast<int>(threadIdx.x) / G;
  const int part = static_cast<int>(threadIdx.x) % G;
  if (j >= sq.lk || part * 8 >= p.d_real) return;
  const long long rows_k = p.rows.cu_k == nullptr ? p.rows.nk : p.rows.total_k;
  const long long kr = static_cast<long long>(sq.k0) + j;
  const long long acc = ((static_cast<long long>(sq.tb) * n_kv + hk) * rows_k + kr) * D + part * 8;
  const long long slice = static_cast<long long>(p.rows_tb) * n_kv * rows_k * D;
  const long long dk_off = sq.tb * p.sdk.b + hk * p.sdk.h + kr * p.sdk.r + part * 8;
  const long long dv_off = sq.tb * p.sdv.b + hk * p.sdv.h + kr * p.sdv.r + part * 8;
  if (!FA_IN_BOUNDS(p.status, acc + (p.split - 1) * slice, 8, p.ext.kvacc) ||
      !FA_IN_BOUNDS(p.status, dk_off, 8, p.ext.dk) || !FA_IN_BOUNDS(p.status, dv_off, 8, p.ext.dv))
    return;
  auto cvt = [&](const float* src, void* dst) {
    float4 x = reinterpret_cast<const float4*>(src)[0], y = reinterpret_cast<const float4*>(src)[1];
    for (int s = 1; s < p.split; ++s) {  // the parts in order
      const float4 u = reinterpret_cast<const float4*>(src + s * slice)[0];
      const float4 t = reinterpret_cast<const float4*>(src + s * slice)[1];
      x = make_float4(x.x + u.x, x.y + u.y, x.z + u.z, x.w + u.w);
      y = make_float4(y.x + t.x, y.y + t.y, y.z + t.z, y.w + t.w);
    }
    *reinterpret_cast<uint4*>(dst) = make_uint4(pack_bf16(x.x, x.y), pack_bf16(x.z, x.w),
                                                pack_bf16(y.x, y.y), pack_bf16(y.z, y.w));
  };
  cvt(p.ws_dk + acc, static_cast<__nv_bfloat16*>(p.dk) + dk_off);
  cvt(p.ws_dv + acc, static_cast<__nv_bfloat16*>(p.dv) + dv_off);
}

// ---------------------------------------------------------------------------
// main kernel
// ---------------------------------------------------------------------------

// GEN: the general instances, which read from the parameters the number of
// query heads per K / V head (grouped-query attention) and the dropout
// counters' row / key offsets (as the forward's POS instances); the others
// see one query head per K / V head and zero offsets at compile time.  Built
// only with the direct mask walk.
template <int D, bool DROPOUT, bool BITS, bool GEN = false>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using L = BwdLayout<D>;
  // Without dropout the P / dS work is split into two phases so that it
  // overlaps the MMAs of neighbouring tiles; with dropout the compute warps
  // are the bottleneck and the serialized order lets the keep-bit generation
  // of the next tile hide under that tile's MMAs instead.
  constexpr bool kTwoPhase = !DROPOUT;
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0 && p.status) atomicExch(p.status, kStatusInternal);
    return;
  }
  auto bar = [&](int i) -> uint32_t { return sbase + L::OFF_BAR + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L::OFF_MISC + 4);
  const WaitGuard g{abort_flag, p.status, p.timeout_ns};
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  BwdWork<BITS> w;
  // d = 256: CTAs 2u and 2u + 1 take the two column halves of unit u
  const int hf = L::RING ? static_cast<int>(blockIdx.x & 1u) : 0;
  const long long unit = L::RING ? static_cast<long long>(blockIdx.x >> 1) : blockIdx.x;
  const int G = GEN ? p.group : 1;  // query heads per K / V head
  const int S = GEN ? p.split : 1;  // parts of a unit (adjacent CTAs)
  const int Gw = G / S;             // query heads one part walks
  const int part = GEN ? static_cast<int>(unit % S) : 0;
  const int n_kv_heads = p.H / G;
  grid_unit(GEN ? unit / S : unit, p.B * n_kv_heads, (p.rows.nk + 127) / 128, p.group_heads,
            &w.bh, &w.kb);  // key tile 0 is heaviest
  w.b = w.bh / n_kv_heads;
  w.hk = w.bh % n_kv_heads;
  const int hq_base = w.hk * G + part * Gw;  // first query head of this part
  {
    const Seq sq = seq_of(p.rows, w.b);
    // a sequence shorter than the longest has no key tile here: leave before
    // any set-up (the whole CTA takes this branch)
    if (w.kb * 128 >= sq.lk) return;
    int kv = sq.lk;
    if (p.seqlens != nullptr && FA_IN_BOUNDS(p.status, w.b, 1, p.ext.seqlens))
      kv = max(0, min(p.seqlens[w.b], sq.lk));
    w.kv_len = kv;
    w.lk = sq.lk;
    w.qrow = sq.q0;
    w.krow = sq.k0;
    w.tb = sq.tb;
    w.off = sq.lk - sq.lq;
    w.nqb = (sq.lq + 127) / 128;
    w.ws0 = ws_row0(p, w.b, hq_base, sq.q0);
  }
  w.alive = w.kb * 128 < w.kv_len;
  w.causal = p.causal != 0;
  if (w.causal) {
    const int lo = w.kb * 128 - w.off;  // first query row that sees this tile's first key
    w.qb_begin = lo <= 0 ? 0 : lo / 128;
  } else {
    w.qb_begin = 0;
  }
  w.nbk = p.nbk;
  w.bm = p.block_mask;
  w.bits = nullptr;
#ifdef FA_DEBUG_BOUNDS
  w.status = p.status;
  w.ext_mask = p.ext.mask;
#endif
  if (BITS && w.bm != nullptr && (w.nqb + 31) / 32 <= L::BIT_WORDS) {
    // every thread takes part: a warp's lanes test 32 consecutive query tiles
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + L::OFF_BITS);
    const int words = (w.nqb + 31) / 32;
    for (int wi = warp; wi < words; wi += kBwdThreads / 32) {
      const int qb = wi * 32 + lane;
      const uint32_t word = __ballot_sync(0xffffffffu, qb < w.nqb && w.act(qb));
      if (lane == 0) bits[wi] = word;
    }
    w.bits = bits;  // read after the __syncthreads below
  }

  if (threadIdx.x == 0) {
    *abort_flag = 0u;
    mbar_init(bar(L::B_KV), 1);
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(bar(L::B_QFULL + s), 1);
      mbar_init(bar(L::B_QEMPTY + s), 1);
    }
    mbar_init(bar(L::B_SFULL), 1);
    mbar_init(bar(L::B_DPFULL), 1);
    mbar_init(bar(L::B_PFULL), 8);     // one arrival per P / dS warp
    mbar_init(bar(L::B_DSFULL), 8);
    mbar_init(bar(L::B_DSEMPTY), 1);
    mbar_init(bar(L::B_DQFULL), 1);
    mbar_init(bar(L::B_DQEMPTY), 4);   // one arrival per dQ warp
    mbar_init(bar(L::B_KVDONE), 1);
    mbar_init(bar(L::B_STAGED), 4);    // one arrival per dQ warp
    if constexpr (L::RING) {
      for (int s = 0; s < 2; ++s) {
        mbar_init(bar(L::B_LDFULL + s), 1);
        mbar_init(bar(L::B_LDEMPTY + s), 8);  // one arrival per P / dS warp
      }
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the walk with this launch's group size and workspace rows per query head
  const long long ws_hs = p.rows.cu_q == nullptr ? p.Npad : p.Rtot;
  auto more = [&](Tile t) { return w.template more<GEN>(t, Gw); };
  auto next_t = [&](Tile t) { return w.template step<GEN>(t); };
  const Tile t_first = w.template first<GEN>(Gw);
  const bool any_work = more(t_first);

  if (warp < 4) {
  if constexpr (L::SPLIT_REGS) setmaxnreg_dec<L::REGS_CTL>();
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0 && any_work) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      tma_prefetch_map(&tm_do);
      mbar_arrive_expect_tx(bar(L::B_KV), 2 * L::TILE);
      for (int pn = 0; pn < L::PANELS; ++pn) {
        tma_load_4d(sbase + L::OFF_K + pn * L::PANEL, &tm_k, bar(L::B_KV), 64 * pn,
                    w.krow + w.kb * 128, w.hk, w.tb);
        tma_load_4d(sbase + L::OFF_V + pn * L::PANEL, &tm_v, bar(L::B_KV), 64 * pn,
                    w.krow + w.kb * 128, w.hk, w.tb);
      }
      if constexpr (L::RING) {
        // Panels in the order the MMA warp consumes them: Q(first), dO(first)
        // for the first S^T / dP^T, then per query tile n: this CTA's two dO
        // panels (dV), Q(n + 1) (next S^T), dO(n + 1) (next dP^T), this CTA's
        // two Q panels (dK).  A tile adds 12 panels (4 for the last), a
        // multiple of the 4 slots, so the pairs for dV and dK always sit in
        // the adjacent slots 0, 1 and 2, 3.  dO(n + 1) takes the slots the
        // next S^T frees early and is resident by the time dP^T(n + 1) can
        // start; the reload of the Q pair waits for dP^T(n + 1) instead, off
        // the path from one tile's dS to the next tile's dP^T.
        int t = 0, nld = 0;
        auto panel = [&](const CUtensorMap* m, int pn, Tile tt) -> bool {
          const int s = t % L::STAGES;
          if (t >= L::STAGES && !mbar_wait(bar(L::B_QEMPTY + s), ((t / L::STAGES) & 1u) ^ 1u, g))
            return false;
          mbar_arrive_expect_tx(bar(L::B_QFULL + s), L::PANEL);
          tma_load_4d(sbase + L::OFF_Q + s * L::PANEL, m, bar(L::B_QFULL + s), 64 * pn,
                      w.qrow + tile_qb<GEN>(tt) * 128, w.template hq<GEN>(tt, hq_base), w.tb);
          ++t;
          return true;
        };
        auto tile4 = [&](const CUtensorMap* m, Tile tt) -> bool {
          for (int pn = 0; pn < L::PANELS; ++pn)
            if (!panel(m, pn, tt)) return false;
          return true;
        };
        auto ld = [&](Tile tt) -> bool {  // -LSE log2e and -D of the tile's rows
          const int s = nld & 1;
          if (nld >= 2 && !mbar_wait(bar(L::B_LDEMPTY + s), ((nld >> 1) & 1u) ^ 1u, g)) return false;
          mbar_arrive_expect_tx(bar(L::B_LDFULL + s), 1024);
          long long roff = w.template wsrow<GEN>(tt, ws_hs);
          if (!FA_IN_BOUNDS(p.status, roff, 128, p.ws_rows)) roff = 0;
          bulk_load(sbase + L::OFF_LD + s * 1024, p.ws_lse2 + roff, 512, bar(L::B_LDFULL + s));
          bulk_load(sbase + L::OFF_LD + s * 1024 + 512, p.ws_delta + roff, 512,
                    bar(L::B_LDFULL + s));
          ++nld;
          return true;
        };
        bool ok = ld(t_first) && tile4(&tm_q, t_first) && tile4(&tm_do, t_first);
        for (Tile tc = t_first; ok && more(tc);) {
          const Tile tn = next_t(tc);
          ok = panel(&tm_do, 2 * hf, tc) && panel(&tm_do, 2 * hf + 1, tc);
          if (ok && more(tn)) ok = ld(tn) && tile4(&tm_q, tn) && tile4(&tm_do, tn);
          if (ok) ok = panel(&tm_q, 2 * hf, tc) && panel(&tm_q, 2 * hf + 1, tc);
          tc = tn;
        }
        if (*abort_flag) {
          for (int j = max(0, t - L::STAGES); j < t; ++j)
            mbar_wait_drain(bar(L::B_QFULL + j % L::STAGES), (j / L::STAGES) & 1u, 100000000ull);
          for (int j = max(0, nld - 2); j < nld; ++j)
            mbar_wait_drain(bar(L::B_LDFULL + (j & 1)), (j >> 1) & 1u, 100000000ull);
          mbar_wait_drain(bar(L::B_KV), 0, 100000000ull);
        }
      } else {
      int it = 0;
      for (Tile tc = t_first; more(tc); tc = next_t(tc), ++it) {
        const int s = it % L::STAGES;
        const uint32_t ph = (it / L::STAGES) & 1u;
        if (it >= L::STAGES && !mbar_wait(bar(L::B_QEMPTY + s), ph ^ 1u, g)) break;
        mbar_arrive_expect_tx(bar(L::B_QFULL + s), 2 * L::TILE + 1024);
        const int hq = w.template hq<GEN>(tc, hq_base);
        for (int pn = 0; pn < L::PANELS; ++pn) {
          tma_load_4d(sbase + L::OFF_Q + s * L::TILE + pn * L::PANEL, &tm_q, bar(L::B_QFULL + s),
                      64 * pn, w.qrow + tile_qb<GEN>(tc) * 128, hq, w.tb);
          tma_load_4d(sbase + L::OFF_DO + s * L::TILE + pn * L::PANEL, &tm_do, bar(L::B_QFULL + s),
                      64 * pn, w.qrow + tile_qb<GEN>(tc) * 128, hq, w.tb);
        }
        long long roff = w.template wsrow<GEN>(tc, ws_hs);
        if (!FA_IN_BOUNDS(p.status, roff, 128, p.ws_rows)) roff = 0;
        bulk_load(sbase + L::OFF_LD + s * 1024, p.ws_lse2 + roff, 512, bar(L::B_QFULL + s));
        bulk_load(sbase + L::OFF_LD + s * 1024 + 512, p.ws_delta + roff, 512, bar(L::B_QFULL + s));
      }
      if (*abort_flag) {
        for (int j = max(0, it - L::STAGES); j < it; ++j)
          mbar_wait_drain(bar(L::B_QFULL + j % L::STAGES), (j / L::STAGES) & 1u, 100000000ull);
        mbar_wait_drain(bar(L::B_KV), 0, 100000000ull);
      }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0 && any_work) {
      constexpr uint32_t kIdS = idesc_bf16(128, 128, false, false);
      constexpr uint32_t kIdKQ = idesc_bf16(128, L::HD, false, true);  // dV, dK
      constexpr uint32_t kIdQ = L::DQ_T ? idesc_bf16(L::HD, 128, true, true)  // dQ^T
                                        : idesc_bf16(128, D, true, true);     // dQ
      const uint32_t k_addr = sbase + L::OFF_K, v_addr = sbase + L::OFF_V;
      // the K panels of this CTA's dQ columns
      const uint32_t kh_addr = k_addr + static_cast<uint32_t>(2 * hf) * L::PANEL;
      const uint32_t ds_addr = sbase + L::OFF_DS;
      bool ok = mbar_wait(bar(L::B_KV), 0, g);

      auto issue_sdp = [&](int s, bool dp_only) {
        const uint32_t q_addr = sbase + L::OFF_Q + s * L::TILE;
        const uint32_t do_addr = sbase + L::OFF_DO + s * L::TILE;
        if (!dp_only) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::PANEL + (kk & 3) * 32;
            mma_ss(tmem + L::COL_S, sdesc_sw128(k_addr + off, 16, 1024),
                   sdesc_sw128(q_addr + off, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(L::B_SFULL));
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::PANEL + (kk & 3) * 32;
            mma_ss(tmem + L::COL_DP, sdesc_sw128(v_addr + off, 16, 1024),
                   sdesc_sw128(do_addr + off, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(L::B_DPFULL));
        }
      };

      // dK += dS^T Q   (A = dS^T K-major in shared memory, B = Q MN-major)
      auto issue_dk = [&](uint32_t q_addr, int it) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + L::COL_DK, sdesc_sw128(ds_addr + (kk >> 2) * L::PANEL + (kk & 3) * 32, 16, 1024),
                 sdesc_sw128(q_addr + kk * 2048, L::PANEL, 1024), kIdKQ,
                 (it > 0 || kk > 0) ? 1u : 0u);
      };
      // dQ_tile = dS K (A = dS MN-major, B = K MN-major), or at d = 128 its
      // transpose dQ^T = K^T dS^T (A = K^T MN-major, B = dS^T MN-major)
      auto issue_dq = [&]() {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ds_desc = sdesc_sw128(ds_addr + kk * 2048, L::PANEL, 1024);
          const uint64_t k_desc = sdesc_sw128(kh_addr + kk * 2048, L::PANEL, 1024);
          if constexpr (L::DQ_T)
            mma_ss(tmem + L::COL_DQ, k_desc, ds_desc, kIdQ, kk > 0 ? 1u : 0u);
          else
            mma_ss(tmem + L::COL_DQ, ds_desc, k_desc, kIdQ, kk > 0 ? 1u : 0u);
        }
      };

      // The MMA warp only needs to know whether a tile remains and whether
      // another follows: the general instances count the steps (G heads times
      // the active query tiles) instead of walking them, which keeps the walk
      // out of this 72-register warp.
      int n_total = 0;
      if constexpr (GEN) {
        for (int qb = w.next(w.qb_begin); qb < w.nqb; qb = w.next(qb + 1)) ++n_total;
        n_total *= Gw;
      }
      auto mma_more = [&](Tile t, int i) { return GEN ? i < n_total : more(t); };
      auto mma_next = [&](Tile t) { return GEN ? t : next_t(t); };
      if constexpr (L::RING) {
        int c = 0;  // panels taken from the ring
        auto slot = [&](int s) -> uint32_t { return sbase + L::OFF_Q + s * L::PANEL; };
        // the slot of the next panel, or -1 once a wait has given up
        auto take = [&]() -> int {
          const int s = c % L::STAGES;
          if (!mbar_wait(bar(L::B_QFULL + s), (c / L::STAGES) & 1u, g)) return -1;
          tc_fence_after();
          ++c;
          return s;
        };
        // this CTA's two panels of dO (for dV) or Q (for dK), in the adjacent
        // slots s, s + 1 (the producer's panel counts keep pairs at even slots)
        auto take_pair = [&]() -> int {
          const int s = take();
          if (s < 0) return -1;
          if ((s & 1) != 0) {
            if (p.status) atomicExch(p.status, kStatusInternal);
            *abort_flag = 1u;
            return -1;
          }
          return take() < 0 ? -1 : s;
        };
        // S^T = K Q^T (dp: dP^T = V dO^T) over the tile's four panels, each
        // slot handed back once its MMAs are done
        auto ring_sdp = [&](bool dp) -> bool {
          const uint32_t a_addr = dp ? v_addr : k_addr;
          const uint32_t col = dp ? L::COL_DP : L::COL_S;
          for (int pn = 0; pn < L::PANELS; ++pn) {
            const int s = take();
            if (s < 0) return false;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tmem + col, sdesc_sw128(a_addr + pn * L::PANEL + kk * 32, 16, 1024),
                     sdesc_sw128(slot(s) + kk * 32, 16, 1024), kIdS, (pn > 0 || kk > 0) ? 1u : 0u);
            mma_commit(bar(L::B_QEMPTY + s));
          }
          mma_commit(bar(dp ? L::B_DPFULL : L::B_SFULL));
          return true;
        };
        // Per query tile: dV, the next tile's S^T (it overwrites S^T / P only
        // after the dV MMAs), then once dS is in shared memory dQ^T, the next
        // tile's dP^T once the dQ^T tile has left its columns, and dK.  Both
        // P / dS orders (two phases, or one under dropout) take the same steps
        // here; without the two phases PFULL already means dS is ready.
        int it = 0;
        if (ok) ok = ring_sdp(false) && ring_sdp(true);
        for (Tile tc = t_first; ok && mma_more(tc, it); ++it) {
          const Tile tn = mma_next(tc);
          if (!mbar_wait(bar(L::B_PFULL), it & 1u, g)) break;
          tc_fence_after();
          const int sd = take_pair();
          if (sd < 0) break;
          // dV += P^T dO   (A = P from TMEM, B = dO's two panels MN-major)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + L::COL_DV, tmem + L::COL_S + 64 * (kk >> 2) + 8 * (kk & 3),
                   sdesc_sw128(slot(sd) + kk * 2048, L::PANEL, 1024), kIdKQ,
                   (it > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(L::B_QEMPTY + sd));
          mma_commit(bar(L::B_QEMPTY + sd + 1));
          if (mma_more(tn, it + 1) && !ring_sdp(false)) break;
          if constexpr (kTwoPhase) {
            if (!mbar_wait(bar(L::B_DSFULL), it & 1u, g)) break;
            tc_fence_after();
          }
          issue_dq();
          mma_commit(bar(L::B_DQFULL));
          if (mma_more(tn, it + 1)) {
            if (!mbar_wait(bar(L::B_DQEMPTY), it & 1u, g)) break;
            tc_fence_after();
            if (!ring_sdp(true)) break;
          }
          const int sq = take_pair();
          if (sq < 0) break;
          issue_dk(slot(sq), it);
          mma_commit(bar(L::B_QEMPTY + sq));
          mma_commit(bar(L::B_QEMPTY + sq + 1));
          mma_commit(bar(L::B_DSEMPTY));
          tc = tn;
        }
      } else {
      int it = 0;
      if (ok) ok = mbar_wait(bar(L::B_QFULL + 0), 0, g);
      if (ok) {
        tc_fence_after();
        issue_sdp(0, false);
        issue_sdp(0, true);
      }
      if constexpr (kTwoPhase) {
        for (Tile tc = t_first; ok && mma_more(tc, it); ++it) {
          const int s = it % L::STAGES;
          const Tile tn = mma_next(tc);
          const int sn = (it + 1) % L::STAGES;
          const uint32_t q_addr = sbase + L::OFF_Q + s * L::TILE;
          const uint32_t do_addr = sbase + L::OFF_DO + s * L::TILE;
          // P of this tile is in TMEM: dV += P^T dO   (A = P from TMEM, B = dO MN-major)
          if (!mbar_wait(bar(L::B_PFULL), it & 1u, g)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + L::COL_DV, tmem + L::COL_S + 64 * (kk >> 2) + 8 * (kk & 3),
                   sdesc_sw128(do_addr + kk * 2048, L::PANEL, 1024), kIdKQ,
                   (it > 0 || kk > 0) ? 1u : 0u);
          // the next tile's S^T overwrites S^T / P only after the dV MMAs above
          if (mma_more(tn, it + 1)) {
            if (!mbar_wait(bar(L::B_QFULL + sn), ((it + 1) / L::STAGES) & 1u, g)) break;
            tc_fence_after();
            issue_sdp(sn, false);
          }
          // dS of this tile is in shared memory: dK and dQ
          if (!mbar_wait(bar(L::B_DSFULL), it & 1u, g)) break;
          tc_fence_after();
          if constexpr (L::DQ_T) {
            // d = 128: dQ^T first, so that its drain out of TMEM runs under
            // the dK MMAs and the next dP^T (same columns) is not kept waiting
            issue_dq();
            mma_commit(bar(L::B_DQFULL));
            issue_dk(q_addr, it);
          } else {
            // d = 64: dK first (the dQ warps stage into this tile's Q / dO
            // stage once the dQ MMAs are done, and dK reads Q from it)
            issue_dk(q_addr, it);
            if (L::SEPARATE_DQ && it > 0) {
              // the dQ columns must have been drained by the previous iteration
              if (!mbar_wait(bar(L::B_DQEMPTY), (it - 1) & 1u, g)) break;
              tc_fence_after();
            }
            issue_dq();
            mma_commit(bar(L::B_DQFULL));
          }
          mma_commit(bar(L::B_DSEMPTY));
          if constexpr (!L::TMA_REDUCE) mma_commit(bar(L::B_QEMPTY + s));
          if (mma_more(tn, it + 1)) {
            // dP^T of the next tile: its columns were read by this tile's dS
            // phase, and (d = 128) hold the dQ tile until it is drained
            if (!L::SEPARATE_DQ) {
              if (!mbar_wait(bar(L::B_DQEMPTY), it & 1u, g)) break;
              tc_fence_after();
            }
            issue_sdp(sn, true);
          }
          tc = tn;
        }
      } else {
        // serialized order, once P and dS are both ready: dV, then the next
        // tile's S^T (it overwrites S^T / P only after the dV MMAs, which
        // execute first) and, at d = 64, its dP^T (the dP^T columns were read
        // by this tile's P / dS warps already), then dK and dQ.  The next
        // tile's S^T / dP^T are ready while dK and dQ still run.  At d = 128
        // the dQ^T tile lives in the dP^T columns, so dP^T comes last.
        for (Tile tc = t_first; ok && mma_more(tc, it); ++it) {
          const int s = it % L::STAGES;
          const Tile tn = mma_next(tc);
          const int sn = (it + 1) % L::STAGES;
          if (!mbar_wait(bar(L::B_PFULL), it & 1u, g)) break;
          tc_fence_after();
          const uint32_t q_addr = sbase + L::OFF_Q + s * L::TILE;
          const uint32_t do_addr = sbase + L::OFF_DO + s * L::TILE;
          // dV += P^T dO   (A = P from TMEM, B = dO MN-major)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + L::COL_DV, tmem + L::COL_S + 64 * (kk >> 2) + 8 * (kk & 3),
                   sdesc_sw128(do_addr + kk * 2048, L::PANEL, 1024), kIdKQ,
                   (it > 0 || kk > 0) ? 1u : 0u);
          if (mma_more(tn, it + 1)) {
            if (!mbar_wait(bar(L::B_QFULL + sn), ((it + 1) / L::STAGES) & 1u, g)) break;
            tc_fence_after();
            issue_sdp(sn, false);
            if (L::SEPARATE_DQ) issue_sdp(sn, true);
          }
          if constexpr (L::DQ_T) {
            // d = 128: dQ^T first (its drain runs under dK, see above)
            issue_dq();
            mma_commit(bar(L::B_DQFULL));
            issue_dk(q_addr, it);
          } else {
            issue_dk(q_addr, it);
            if (L::SEPARATE_DQ && it > 0) {
              // the dQ columns must have been drained by the previous iteration
              if (!mbar_wait(bar(L::B_DQEMPTY), (it - 1) & 1u, g)) break;
              tc_fence_after();
            }
            issue_dq();
            mma_commit(bar(L::B_DQFULL));
          }
          mma_commit(bar(L::B_DSEMPTY));
          if constexpr (!L::TMA_REDUCE) mma_commit(bar(L::B_QEMPTY + s));
          if (!L::SEPARATE_DQ && mma_more(tn, it + 1)) {
            if (!mbar_wait(bar(L::B_DQEMPTY), it & 1u, g)) break;
            tc_fence_after();
            issue_sdp(sn, true);
          }
          tc = tn;
        }
      }
      }
      mma_commit(bar(L::B_KVDONE));
      mbar_wait_drain(bar(L::B_KVDONE), 0, 1000000000ull);
    }
  }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------ P / dS warpgroups
    const int wg = (warp - 4) >> 2;
    const int wq = warp & 3;
    const int j = wq * 32 + lane;  // key row within the tile
    const int jg = w.kb * 128 + j;
    const bool key_live = jg < w.kv_len;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
    const float2 rs2 = make_float2(p.drop_rscale, p.drop_rscale);
    bool ok = true;
    int it = 0;
    for (Tile tc = t_first; more(tc); tc = next_t(tc), ++it) {
      const int qb = tile_qb<GEN>(tc);
      const int s = it % L::STAGES;
      // Dropout keep bits of this key for the warpgroup's 64 queries, drawn
      // before the waits (they do not depend on S or dP).  A block covers
      // eight keys, which are the eight lanes of an aligned group: lane r of
      // the group computes the block of query q0 + 8 g + r, then the eight
      // 32-bit masks are exchanged and shifted so that every lane holds its
      // own key's bits: keep(query qoff + 8 g + r) = bit 8 g of kw[c][r].
      uint32_t kw[2][8];
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int r = 0; r < 8; ++r) kw[c][r] = 0u;
      if constexpr (DROPOUT) {
        const uint32_t thr = p.drop_threshold;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int qoff = 64 * wg + 32 * c;
          uint32_t own = 0u;
#pragma unroll
          for (int gq = 0; gq < 4; ++gq) {
            const uint32_t qg = (GEN ? p.drop_row0 : 0u) +
                                static_cast<uint32_t>(qb * 128 + qoff + 8 * gq + (lane & 7));
            const Philox4 rnd = philox4x32_10((GEN ? p.drop_kgrp0 : 0u) + static_cast<uint32_t>(jg >> 3), qg,
                                              static_cast<uint32_t>(w.template hq<GEN>(tc, hq_base)), static_cast<uint32_t>(w.b),
                                              p.rk);
            own |= keep_byte(rnd, thr) << (8 * gq);
          }
#pragma unroll
          for (int r = 0; r < 8; ++r)
            kw[c][r] = __shfl_sync(0xffffffffu, own, (lane & ~7) | r) >> (lane & 7);
        }
      }
      // the LSE / D slices come with the Q / dO stage, or (ring) on their own
      const int ls = L::RING ? (it & 1) : s;
      if constexpr (L::RING)
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_LDFULL + ls), (it >> 1) & 1u, g));
      else
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_QFULL + s), (it / L::STAGES) & 1u, g));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_SFULL), it & 1u, g));
      // -LSE log2e and -D of the tile's 128 queries
      const float* nlse = reinterpret_cast<const float*>(smem + L::OFF_LD + ls * 1024);
      const float* ndlt = nlse + 128;
      // causal: query q of this tile sees this thread's key iff q >= qmin
      const bool diag = w.causal && (w.kb * 128 + 127 > qb * 128 + w.off);
      const int qmin = j + (w.kb - qb) * 128 - w.off;
      // only the diagonal tile of a causal mask and padding keys need masking;
      // the choice must be warp-uniform (the TMEM loads and stores in both
      // versions are warp-collective)
      const bool masked = __any_sync(0xffffffffu, diag || !key_live);

      // P for queries qoff + 4 k4 + [0, 4) of this key: exp2(S^T scale log2e - LSE log2e)
      auto p_quad = [&](auto mask_tag, const uint32_t* sv, int qoff, int k4, float pv[4]) {
        constexpr bool MASKED = decltype(mask_tag)::value;
        const float4 lv = reinterpret_cast<const float4*>(nlse + qoff)[k4];
        const float2 x01 = fma2(make_float2(__uint_as_float(sv[4 * k4]), __uint_as_float(sv[4 * k4 + 1])),
                                sl2, make_float2(lv.x, lv.y));
        const float2 x23 = fma2(make_float2(__uint_as_float(sv[4 * k4 + 2]), __uint_as_float(sv[4 * k4 + 3])),
                                sl2, make_float2(lv.z, lv.w));
        pv[0] = fast_exp2(x01.x);
        pv[1] = fast_exp2(x01.y);
        pv[2] = fast_exp2(x23.x);
        pv[3] = fast_exp2(x23.y);
        if constexpr (MASKED) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (!key_live || (diag && qoff + 4 * k4 + e < qmin)) pv[e] = 0.f;
        }
      };
      // keep bit of query qoff + 4 k4 + e (= 8 g + r, g = k4 / 2, r = 4 (k4 % 2) + e)
      auto keep_of = [&](int c, int k4, int e) -> bool {
        return (kw[c][4 * (k4 & 1) + e] & (1u << (8 * (k4 >> 1)))) != 0u;
      };

      if constexpr (kTwoPhase) {
        if (!ok) break;
        tc_fence_after();

        // ---- P phase: the dropped P goes to TMEM for dV, the undropped P is
        // kept as fp16 pairs (P <= 1 here) for the dS phase, negated where
        // dropout drops the pair (P >= 0, and a P of 0 contributes nothing
        // either way).
        uint32_t pu[32];
        auto p_phase = [&](auto mask_tag) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int qoff = 64 * wg + 32 * c;  // query offset within the tile
            uint32_t sv[32];
            tmem_ld32<0>(lane_addr + L::COL_S + qoff, sv);
            tmem_wait_ld32<0>(sv);
            uint32_t ppk[16];
#pragma unroll
            for (int k4 = 0; k4 < 8; ++k4) {
              float pv[4], pe[4], pk4[4];
              p_quad(mask_tag, sv, qoff, k4, pv);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                pe[e] = pv[e];
                pk4[e] = pv[e];
                if constexpr (DROPOUT) {
                  const bool keep = keep_of(c, k4, e);
                  pe[e] = keep ? pv[e] : 0.f;
                  pk4[e] = keep ? pv[e] : -pv[e];
                }
              }
              ppk[2 * k4] = pack_bf16(pe[0], pe[1]);
              ppk[2 * k4 + 1] = pack_bf16(pe[2], pe[3]);
              pu[16 * c + 2 * k4] = pack_f16(pk4[0], pk4[1]);
              pu[16 * c + 2 * k4 + 1] = pack_f16(pk4[2], pk4[3]);
            }
            // P^T (bf16 pairs) into TMEM: queries [64 wg, 64 wg + 64) -> columns
            // [64 wg, 64 wg + 32), inside this warpgroup's S^T columns already read
            tmem_st16<0>(lane_addr + L::COL_S + 64 * wg + 16 * c, ppk);
          }
        };
        if (masked) p_phase(std::true_type{});
        else p_phase(std::false_type{});
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::B_PFULL));

        // ---- dS phase: dS = P (dP - D), dP = dP_drop * keep / q under dropout
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_DPFULL), it & 1u, g));
        if (ok && it > 0)
          ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_DSEMPTY), (it - 1) & 1u, g));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int qoff = 64 * wg + 32 * c;
          uint32_t dv[32];
          tmem_ld32<0>(lane_addr + L::COL_DP + qoff, dv);
          tmem_wait_ld32<0>(dv);
          const float2* d2 = reinterpret_cast<const float2*>(ndlt + qoff);
          uint32_t dpk[16];
#pragma unroll
          for (int k2 = 0; k2 < 16; ++k2) {
            float2 pv = unpack_f16(pu[16 * c + k2]);
            float2 dp = make_float2(__uint_as_float(dv[2 * k2]), __uint_as_float(dv[2 * k2 + 1]));
            float2 t;
            if constexpr (DROPOUT) {
              // negative P: dropped
              dp.x = (pv.x >= 0.f) ? dp.x : 0.f;
              dp.y = (pv.y >= 0.f) ? dp.y : 0.f;
              pv = make_float2(fabsf(pv.x), fabsf(pv.y));
              t = fma2(dp, rs2, d2[k2]);
            } else {
              t = add2(dp, d2[k2]);
            }
            const float2 ds = mul2(pv, t);
            dpk[k2] = pack_bf16(ds.x, ds.y);
          }
          // dS^T row j into the 128-byte-swizzled [keys][queries] buffer, panel wg
          const uint32_t row_addr = sbase + L::OFF_DS + wg * L::PANEL + j * 128;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            const uint32_t chunk = static_cast<uint32_t>(4 * c + ch) ^ static_cast<uint32_t>(j & 7);
            st_shared_v4(row_addr + chunk * 16, dpk[4 * ch], dpk[4 * ch + 1], dpk[4 * ch + 2],
                         dpk[4 * ch + 3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(L::B_DSFULL));
          if constexpr (L::RING) mbar_arrive(bar(L::B_LDEMPTY + ls));  // LSE / D read
        }
      } else {
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_DPFULL), it & 1u, g));
        if (ok && it > 0)
          ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_DSEMPTY), (it - 1) & 1u, g));
        if (!ok) break;
        tc_fence_after();
        auto both = [&](auto mask_tag) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int qoff = 64 * wg + 32 * c;  // query offset within the tile
            uint32_t sv[32], dv[32];
            tmem_ld32<0>(lane_addr + L::COL_S + qoff, sv);
            tmem_ld32<0>(lane_addr + L::COL_DP + qoff, dv);
            tmem_wait_ld32<0>(sv);
            tmem_wait_ld32<0>(dv);
            const float4* d4 = reinterpret_cast<const float4*>(ndlt + qoff);
            uint32_t ppk[16], dpk[16];
#pragma unroll
            for (int k4 = 0; k4 < 8; ++k4) {
              float pv[4], pe[4], dp[4];
              p_quad(mask_tag, sv, qoff, k4, pv);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                pe[e] = pv[e];
                dp[e] = __uint_as_float(dv[4 * k4 + e]);
                if constexpr (DROPOUT) {
                  const bool keep = keep_of(c, k4, e);
                  pe[e] = keep ? pv[e] : 0.f;
                  dp[e] = keep ? dp[e] : 0.f;
                }
              }
              const float4 dl = d4[k4];
              float2 t01, t23;
              if constexpr (DROPOUT) {
                t01 = fma2(make_float2(dp[0], dp[1]), rs2, make_float2(dl.x, dl.y));
                t23 = fma2(make_float2(dp[2], dp[3]), rs2, make_float2(dl.z, dl.w));
              } else {
                t01 = add2(make_float2(dp[0], dp[1]), make_float2(dl.x, dl.y));
                t23 = add2(make_float2(dp[2], dp[3]), make_float2(dl.z, dl.w));
              }
              const float2 ds01 = mul2(make_float2(pv[0], pv[1]), t01);
              const float2 ds23 = mul2(make_float2(pv[2], pv[3]), t23);
              ppk[2 * k4] = pack_bf16(pe[0], pe[1]);
              ppk[2 * k4 + 1] = pack_bf16(pe[2], pe[3]);
              dpk[2 * k4] = pack_bf16(ds01.x, ds01.y);
              dpk[2 * k4 + 1] = pack_bf16(ds23.x, ds23.y);
            }
            // P^T (bf16 pairs) into TMEM: queries [64 wg, 64 wg + 64) -> columns [64 wg, 64 wg + 32)
            tmem_st16<0>(lane_addr + L::COL_S + 64 * wg + 16 * c, ppk);
            // dS^T row j into the 128-byte-swizzled [keys][queries] buffer, panel wg
            const uint32_t row_addr = sbase + L::OFF_DS + wg * L::PANEL + j * 128;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              const uint32_t chunk = static_cast<uint32_t>(4 * c + ch) ^ static_cast<uint32_t>(j & 7);
              st_shared_v4(row_addr + chunk * 16, dpk[4 * ch], dpk[4 * ch + 1], dpk[4 * ch + 2],
                           dpk[4 * ch + 3]);
            }
          }
        };
        if (masked) both(std::true_type{});
        else both(std::false_type{});
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(L::B_PFULL));
          if constexpr (L::RING) mbar_arrive(bar(L::B_LDEMPTY + ls));  // LSE / D read
        }
      }
    }

    // -------------------------------------------------- dK, dV epilogue
    const int n_it = it;
    if (ok && any_work) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_KVDONE), 0, g));
    if (ok) {
      tc_fence_after();
      const bool row_ok = jg < w.lk;
      const long long kr = w.krow + jg;
#pragma unroll
      for (int c = 0; c < L::HD / 64; ++c) {
        const int tcol = wg * (L::HD / 2) + 32 * c;  // TMEM column of this CTA's slice
        const int col = L::HD * hf + tcol;            // feature column
        uint32_t a[32], bk[32];
        if (any_work && n_it > 0) {
          tmem_ld32<0>(lane_addr + L::COL_DV + tcol, a);
          tmem_ld32<0>(lane_addr + L::COL_DK + tcol, bk);
          tmem_wait_ld32<0>(a);
          tmem_wait_ld32<0>(bk);
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) a[k] = bk[k] = 0u;
        }
        const long long dv_off = w.tb * p.sdv.b + w.hk * p.sdv.h + kr * p.sdv.r + col;
        const long long dk_off = w.tb * p.sdk.b + w.hk * p.sdk.h + kr * p.sdk.r + col;
        if (GEN && S > 1) {
          // one part of a split unit: its (scaled) dK / dV go to its own fp32
          // slice ([part][tb][H_kv][key rows][D]); the conversion sums the
          // slices in part order, so the result does not depend on timing
          const long long rows_k = p.rows.cu_k == nullptr ? p.rows.nk : p.rows.total_k;
          const long long acc =
              (((static_cast<long long>(part) * p.rows_tb + w.tb) * n_kv_heads + w.hk) * rows_k +
               kr) * D + col;
          if (row_ok && col < p.d_real && FA_IN_BOUNDS(p.status, acc, 32, p.ext.kvacc)) {
            float4* dvp = reinterpret_cast<float4*>(p.ws_dv + acc);
            float4* dkp = reinterpret_cast<float4*>(p.ws_dk + acc);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float rs = p.drop_rscale, sc = p.scale;
              dvp[k] = make_float4(__uint_as_float(a[4 * k]) * rs, __uint_as_float(a[4 * k + 1]) * rs,
                                   __uint_as_float(a[4 * k + 2]) * rs, __uint_as_float(a[4 * k + 3]) * rs);
              dkp[k] = make_float4(__uint_as_float(bk[4 * k]) * sc, __uint_as_float(bk[4 * k + 1]) * sc,
                                   __uint_as_float(bk[4 * k + 2]) * sc,
                                   __uint_as_float(bk[4 * k + 3]) * sc);
            }
          }
        } else if (row_ok && col < p.d_real && FA_IN_BOUNDS(p.status, dv_off, 32, p.ext.dv) &&
                   FA_IN_BOUNDS(p.status, dk_off, 32, p.ext.dk)) {
          uint4* dvp = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dv) + dv_off);
          uint4* dkp = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dk) + dk_off);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint32_t vv[4], kk4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int x = 8 * k + 2 * e;
              vv[e] = pack_bf16(__uint_as_float(a[x]) * p.drop_rscale,
                                __uint_as_float(a[x + 1]) * p.drop_rscale);
              kk4[e] = pack_bf16(__uint_as_float(bk[x]) * p.scale, __uint_as_float(bk[x + 1]) * p.scale);
            }
            dvp[k] = make_uint4(vv[0], vv[1], vv[2], vv[3]);
            dkp[k] = make_uint4(kk4[0], kk4[1], kk4[2], kk4[3]);
          }
        }
      }
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------- dQ reduction
    if constexpr (L::SPLIT_REGS) setmaxnreg_inc<L::REGS_DQ>();
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // query row within the tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    int it = 0;
    bool issued = false;
    for (Tile tc = t_first; more(tc); tc = next_t(tc), ++it) {
      const int s = it % L::STAGES;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_DQFULL), it & 1u, g))) break;
      tc_fence_after();
      // box b (columns 32 b .. 32 b + 31) of the staging area: the Q buffer of
      // stage s holds the first D / 64 boxes, its dO buffer the rest
      auto box = [&](int b) -> uint32_t {
        return b < L::PANELS ? sbase + L::OFF_Q + s * L::TILE + b * L::PANEL
                             : sbase + L::OFF_DO + s * L::TILE + (b - L::PANELS) * L::PANEL;
      };
      if constexpr (L::DQ_T) {
        // lane r = feature HD hf + r; column c = query qb * 128 + c: each
        // warp's reduction covers 32 consecutive floats of one accumulator
        // row.  The whole tile comes out of TMEM first and its columns go back
        // to the MMA warp (for the next tile's dP^T) before the reductions.
        const int feat = L::HD * hf + r;
        float* dst = p.ws_dq + w.template wsrow<GEN>(tc, ws_hs) * D + feat;
        uint32_t a[128];
        tmem_ld32<0>(lane_addr + L::COL_DQ + 0, a);
        tmem_ld32<32>(lane_addr + L::COL_DQ + 32, a);
        tmem_ld32<64>(lane_addr + L::COL_DQ + 64, a);
        tmem_ld32<96>(lane_addr + L::COL_DQ + 96, a);
        tmem_wait_ld32<0>(a);
        tmem_wait_ld32<32>(a);
        tmem_wait_ld32<64>(a);
        tmem_wait_ld32<96>(a);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::B_DQEMPTY));  // the dQ columns of TMEM are free again
        // features past d (zero columns of d = 96 / 192) are left out, whole
        // warps at a time (d is a multiple of 32)
        // (the tile's rows are consecutive: its first and last accumulator
        // element bound every one it touches)
        const long long acc0 = w.template wsrow<GEN>(tc, ws_hs) * D + feat;
        if (feat < p.d_real && FA_IN_BOUNDS(p.status, acc0, 127ll * D + 1, p.ws_rows * D)) {
#pragma unroll
          for (int k = 0; k < 128; ++k) red_add_f32(dst + k * D, __uint_as_float(a[k]));
        }
      } else {
        // lane r = query r; columns 32 b .. 32 b + 31 = box b
#pragma unroll
        for (int b = 0; b < D / 32; ++b) {
          uint32_t a[32];
          tmem_ld32<0>(lane_addr + L::COL_DQ + 32 * b, a);
          tmem_wait_ld32<0>(a);
          const uint32_t row = box(b) + r * 128;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            st_shared_v4(row + ((k ^ (r & 7)) << 4), a[4 * k], a[4 * k + 1], a[4 * k + 2], a[4 * k + 3]);
        }
      }
      if constexpr (!L::DQ_T) {
        tc_fence_before();
        if constexpr (L::TMA_REDUCE) fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(L::B_DQEMPTY));  // the dQ columns of TMEM are free again
          if constexpr (L::TMA_REDUCE) mbar_arrive(bar(L::B_STAGED));
        }
      }
      if (L::TMA_REDUCE && warp == 12) {
        // one thread reduces the staged tile into the accumulators, then hands
        // the stage back to the producer once the boxes have been read
        bool staged = true;
        if (lane == 0) {
          staged = mbar_wait(bar(L::B_STAGED), it & 1u, g);
          if (staged) {
            const int32_t y = static_cast<int32_t>(w.template wsrow<GEN>(tc, ws_hs));
#pragma unroll
            for (int b = 0; b < D / 32; ++b) tma_reduce_add_2d(&tm_dq, box(b), 32 * b, y);
            bulk_commit_group();
            bulk_wait_group_read0();
            issued = true;
            mbar_arrive(bar(L::B_QEMPTY + s));
          }
        }
        if (!__shfl_sync(0xffffffffu, staged ? 1 : 0, 0)) break;  // the whole warp leaves
      }
    }
    if (issued) bulk_wait_group0();  // the reductions have landed before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// (row blocks of the longest sequence rounded up to 128 rows) x (B * H)
template <int D>
dim3 prepost_grid(const BwdParams& p) {
  const long long rows = (static_cast<long long>(p.rows.nq) + 127) / 128 * 128;
  return dim3(static_cast<unsigned>(rows / kRowsPerBlock<D>), static_cast<unsigned>(p.B * p.H), 1);
}

template <int D>
cudaError_t launch_pre_t(const BwdParams& p, cudaStream_t stream) {
  return launch_overlapped(bwd_pre_kernel<D>, prepost_grid<D>(p), dim3(256), 0, stream, p);
}

template <int D, bool DROPOUT, bool BITS, bool GEN = false>
cudaError_t launch_main_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tdo, const CUtensorMap& tdq, const BwdParams& p,
                          cudaStream_t stream) {
  using L = BwdLayout<D>;
  static_assert(!BITS || L::BIT_WORDS > 0, "no bitmask at this head dim");
  auto kern = bwd_main_kernel<D, DROPOUT, BITS, GEN>;
  // The setmaxnreg split (d = 128) is sized for exactly 128 registers per
  // thread at launch; with any other count an increase could wait forever.
  static OncePerContext prepared;
  cudaError_t e = prepared.run([&]() -> cudaError_t {
    if constexpr (L::SPLIT_REGS) {
      cudaFuncAttributes attr{};
      cudaError_t r = cudaFuncGetAttributes(&attr, kern);
      if (r != cudaSuccess) return r;
      if (attr.numRegs != 128) return cudaErrorInvalidConfiguration;
    }
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(L::SMEM));
  });
  if (e != cudaSuccess) return e;
  // one unit per (b, K / V head, key tile); d = 256: two CTAs (column halves) each
  const long long ctas = static_cast<long long>((p.rows.nk + 127) / 128) * p.B *
                         (p.H / (GEN ? p.group : 1)) * (GEN ? p.split : 1) * (L::RING ? 2 : 1);
  if (ctas > 0x7FFFFFFFll) return cudaErrorInvalidConfiguration;
  return launch_overlapped(kern, dim3(static_cast<unsigned>(ctas)), dim3(kBwdThreads), L::SMEM,
                           stream, tq, tk, tv, tdo, tdq, p);
}

template <int D>
cudaError_t launch_post_t(const BwdParams& p, cudaStream_t stream) {
  return launch_overlapped(bwd_post_kernel<D>, prepost_grid<D>(p), dim3(256), 0, stream, p);
}

}  // namespace

cudaError_t launch_bwd_pre(int d, const BwdParams& p, cudaStream_t stream) {
  if (d == 64) return launch_pre_t<64>(p, stream);
  if (d == 128) return launch_pre_t<128>(p, stream);
  if (d == 256) return launch_pre_t<256>(p, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_main(int d, bool dropout, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, const CUtensorMap& tdo, const CUtensorMap& tdq,
                            const BwdParams& p, cudaStream_t stream) {
  // grouped K / V heads, or dropout on a block of a longer sequence
  if (p.group > 1 || (dropout && (p.drop_row0 != 0u || p.drop_kgrp0 != 0u))) {
    if (d == 64)
      return dropout ? launch_main_t<64, true, false, true>(tq, tk, tv, tdo, tdq, p, stream)
                     : launch_main_t<64, false, false, true>(tq, tk, tv, tdo, tdq, p, stream);
    if (d == 128)
      return dropout ? launch_main_t<128, true, false, true>(tq, tk, tv, tdo, tdq, p, stream)
                     : launch_main_t<128, false, false, true>(tq, tk, tv, tdo, tdq, p, stream);
    if (d == 256)
      return dropout ? launch_main_t<256, true, false, true>(tq, tk, tv, tdo, tdq, p, stream)
                     : launch_main_t<256, false, false, true>(tq, tk, tv, tdo, tdq, p, stream);
    return cudaErrorInvalidValue;
  }
  if (d == 64) {
    // a block mask whose columns fit the bitmask (the CTAs' query tiles are
    // below the longest sequence's)
    const bool bits = p.block_mask != nullptr && p.mask_bitmap != 0 &&
                      ((p.rows.nq + 127) / 128 + 31) / 32 <= BwdLayout<64>::BIT_WORDS;
    if (bits)
      return dropout ? launch_main_t<64, true, true>(tq, tk, tv, tdo, tdq, p, stream)
                     : launch_main_t<64, false, true>(tq, tk, tv, tdo, tdq, p, stream);
    return dropout ? launch_main_t<64, true, false>(tq, tk, tv, tdo, tdq, p, stream)
                   : launch_main_t<64, false, false>(tq, tk, tv, tdo, tdq, p, stream);
  }
  if (d == 128) return dropout ? launch_main_t<128, true, false>(tq, tk, tv, tdo, tdq, p, stream)
                               : launch_main_t<128, false, false>(tq, tk, tv, tdo, tdq, p, stream);
  if (d == 256) return dropout ? launch_main_t<256, true, false>(tq, tk, tv, tdo, tdq, p, stream)
                               : launch_main_t<256, false, false>(tq, tk, tv, tdo, tdq, p, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_kv_post(int d, const BwdParams& p, cudaStream_t stream) {
  const long long rows = (static_cast<long long>(p.rows.nk) + 127) / 128 * 128;
  auto grid = [&](int rpb) {
    return dim3(static_cast<unsigned>(rows / rpb), static_cast<unsigned>(p.B * (p.H / p.group)), 1);
  };
  if (d == 64) return launch_overlapped(bwd_kv_post_kernel<64>, grid(kRowsPerBlock<64>), dim3(256), 0, stream, p);
  if (d == 128) return launch_overlapped(bwd_kv_post_kernel<128>, grid(kRowsPerBlock<128>), dim3(256), 0, stream, p);
  if (d == 256) return launch_overlapped(bwd_kv_post_kernel<256>, grid(kRowsPerBlock<256>), dim3(256), 0, stream, p);
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_post(int d, const BwdParams& p, cudaStream_t stream) {
  if (d == 64) return launch_post_t<64>(p, stream);
  if (d == 128) return launch_post_t<128>(p, stream);
  if (d == 256) return launch_post_t<256>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace fa
