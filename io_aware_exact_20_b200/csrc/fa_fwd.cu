// Forward pass of exact attention on sm_100a.
//
// Work unit: one (b, h) and NQ 128-row Q tiles (NQ = 2 at d = 128, 1 at
// d = 64 and 256) that share every K/V tile the CTA loads.  The CTA walks the K/V tiles
// of its head that at least one of its Q tiles needs (tiles that are fully
// masked by the causal mask, the key lengths or the block mask are neither
// loaded nor computed).
//
// Each Q tile is processed by KS softmax streams (KS = 2 at d = 64, else 1);
// with KS = 2, stream h of a Q tile owns keys [128 kb + 64 h, 128 kb + 64 h + 64)
// of every K/V tile kb, with KS = 1 the whole tile, and each stream keeps its
// own running maximum, row sum and O accumulator.  Per K/V tile and active
// stream:
//
//   S = Q_t K_h^T           tcgen05.mma, bf16 x bf16 -> fp32 in TMEM
//   P = exp2(S * scale * log2e - m)   online softmax, one thread per row
//   O_h += P V_h            tcgen05.mma with P read from TMEM
//
// and at the end the streams of a Q tile merge: with M = max_h m_h,
// O = sum_h 2^(m_h - M) O_h / sum_h 2^(m_h - M) l_h (the softmax of a key range
// split in two, recombined from per-part statistics as in the pages' tiling
// section).  The d = 64 forward is limited by how well the softmax warps hide
// their latencies, and the split gives each SM sub-partition more of them; at
// d = 128 the O accumulators leave no TMEM for it.
//
// Roles:
//   warp 0            TMA producer: Q tiles once, then K/V tiles into a ring
//                     (d = 256: K tiles only)
//   warp 1            TMEM allocator and single-thread MMA issuer
//   warp 2            d = 256: TMA producer of the V tiles; else idle
//   warp 3            idle
//   warpgroup 1 + s   softmax stream s (thread = row, TMEM lanes 0..127)
//
// The running maximum m is only moved when a new block raises it by more than
// 8 (in log2 units); until then exp2 values may reach 2^8, and O and the row
// sum l keep using the same stale maximum, so the final O / l and
// LSE = ln2 * (m + log2 l) are unchanged (the online-softmax rescaling of the
// tiling section of the pages, applied lazily).
//
// TMEM columns: S/P of stream s at [KW s, KW s + KW) (KW = 128 / KS keys; P
// packed as bf16 pairs in the first KW / 2 columns), O of stream s at
// [KW NS + D s, KW NS + D s + D), NS = NQ KS streams.  d = 256: S/P of tile n
// at [128 (n & 1), 128 (n & 1) + 128) (two buffers), O at [256, 512).
#include <cuda_bf16.h>

#include "devctx.h"
#include "kernels.h"
#include "philox.cuh"
#include "ptx.cuh"

namespace fa {
namespace {

constexpr float kLn2 = 0.693147180559945309f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// Per head dimension:
//   d = 128: two Q tiles per CTA (NQ = 2) share every K/V tile, one softmax
//            stream each (KS = 1); the four accumulators fill TMEM.
//   d = 64:  one Q tile per CTA (NQ = 1) and two CTAs per SM, the tile's keys
//            split between two softmax streams (KS = 2): four softmax
//            warpgroups per SM either way, but each CTA walks only the K/V
//            tiles its own Q tile needs (which matters under block masks) and
//            one CTA's set-up and epilogue hide under the other's main loop.
//   d = 256 (WIDE, also d = 192 with zero columns): one Q tile per CTA and
//            one softmax stream; S (128 columns) and O (256) take 384 TMEM
//            columns and a 64 KB Q tile plus one 128 KB K/V stage most of the
//            shared memory, so K and V are released separately (K once its S
//            MMA is done, V once its PV MMA is done) and the next tile's K
//            loads while this tile's softmax runs.  No register split: the
//            256 threads can hold 255 registers each.
template <int D>
struct FwdCfg {
  static constexpr bool WIDE = D == 256;
  static constexpr int NQ = D == 128 ? 2 : 1;  // Q tiles per CTA
  static constexpr int KS = D == 64 ? 2 : 1;   // softmax streams per Q tile
  static constexpr int NS = NQ * KS;           // softmax streams = softmax warpgroups
  static constexpr int KW = 128 / KS;          // keys per stream per K/V tile
  static constexpr int THREADS = 128 * (1 + NS);
  static constexpr int MIN_BLOCKS = D == 64 ? 2 : 1;
  static constexpr bool SPLIT_REGS = !WIDE;
  // registers per thread at launch (checked before the first launch): the
  // largest multiple of 8 that MIN_BLOCKS CTAs of THREADS threads can hold
  static constexpr int LAUNCH_REGS = (65536 / (THREADS * MIN_BLOCKS)) & ~7;
  // setmaxnreg moves registers from warpgroup 0 (producer, MMA issuer) to the
  // softmax warpgroups, within the THREADS x LAUNCH_REGS of the launch
  static constexpr uint32_t REGS_CTL = KS == 1 ? 72 : 32;
  static constexpr uint32_t REGS_SOFTMAX =
      SPLIT_REGS ? ((THREADS * LAUNCH_REGS - 128 * REGS_CTL) / (128 * NS)) & ~7u : 248u;
  static constexpr int MAX_PARTS = KW == 128 ? 8 : 4;  // max / sum chains per row
  static_assert(!SPLIT_REGS || 128 * (REGS_CTL + NS * REGS_SOFTMAX) <= THREADS * LAUNCH_REGS,
                "register split exceeds the launch allocation");
  static_assert(!SPLIT_REGS || (REGS_SOFTMAX <= 256 && REGS_SOFTMAX >= 96),
                "softmax register budget");
};

template <int D>
struct FwdLayout {
  using C = FwdCfg<D>;
  static constexpr int NQ = C::NQ;
  static constexpr int PANELS = D / 64;                 // 64-column, 128-byte-swizzled panels
  static constexpr uint32_t PANEL = 128u * 128u;        // bytes of one [128 rows][64 cols] panel
  static constexpr uint32_t TILE = PANEL * PANELS;      // bytes of one 128-row tile
  static constexpr int STAGES = C::WIDE ? 1 : 2;        // K/V ring depth
  // K and V of a stage released by separate barriers (else one, after PV)
  static constexpr bool SPLIT_RELEASE = C::WIDE;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_KV = NQ * TILE;
  static constexpr uint32_t OFF_XCH = OFF_KV + STAGES * 2 * TILE;  // [NS][128] (m, l) for the merge
  static constexpr uint32_t OFF_BAR = OFF_XCH + (C::KS > 1 ? C::NS * 128 * 8 : 0);
  static constexpr int B_QFULL = 0;
  static constexpr int B_KFULL = 2;
  static constexpr int B_VFULL = B_KFULL + STAGES;
  static constexpr int B_KVEMPTY = B_VFULL + STAGES;  // with SPLIT_RELEASE: K released
  static constexpr int B_VEMPTY = B_KVEMPTY + STAGES;  // with SPLIT_RELEASE: V released
  // S / P buffers per stream: two in the WIDE kernel, so that the next tile's
  // S is computed while this tile's softmax runs (its TMEM has room: 2 x 128
  // S columns + 256 O columns)
  static constexpr int S_BUFS = C::WIDE ? 2 : 1;
  static constexpr int B_SFULL = B_KVEMPTY + STAGES * (SPLIT_RELEASE ? 2 : 1);  // per stream, buffer
  static constexpr int B_PFULL = B_SFULL + C::NS * S_BUFS;  // per stream
  static constexpr int B_ODONE = B_PFULL + C::NS;     // per stream
  static constexpr int B_DRAIN = B_ODONE + C::NS;
  static constexpr int NBAR = B_DRAIN + 1;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
  // block masks: per Q tile a bitmask of the K/V tiles it takes part in
  // (BIT_WORDS / NQ words each, so up to 32768 / NQ key tiles)
  static constexpr int BIT_WORDS = 1024;
  static constexpr uint32_t OFF_BITS = OFF_MISC + 16;
  static constexpr uint32_t SMEM = OFF_BITS + BIT_WORDS * 4;
  static constexpr uint32_t O_COL = C::KW * C::NS * S_BUFS;
  static constexpr uint32_t TMEM_COLS = O_COL + C::NS * D <= 256 ? 256 : 512;
  static_assert(SMEM <= (C::MIN_BLOCKS == 1 ? 232448u : 113u * 1024u), "shared memory budget");
  static_assert(O_COL + C::NS * D <= TMEM_COLS, "TMEM budget");
};

// Which (Q tile, K/V tile) pairs of this CTA take part.  Rows and keys are
// counted inside the CTA's sequence; qrow / krow are the tensor rows of the
// sequence's first query / key and tb its batch coordinate.  Under the causal
// mask query i sees key j iff j <= i + off, off = (keys) - (queries) of the
// sequence (bottom-right alignment).
//
// Under a block mask the CTA first gathers, for each of its Q tiles, the K/V
// tiles below kb_end that take part into a bitmask in shared memory (one
// coalesced pass over the mask row); every role then finds its next tile with
// a word read and a find-first-set instead of testing the mask's bytes one by
// one.  kRows bitmask rows (one per Q tile) of kWpr words each; kernels
// launched without a block mask, or with rows longer than the bitmask, are
// built without it (kBits false) and test the mask's bytes directly.
template <int kRows, int kWpr, bool kBits>
struct FwdWork {
  int b, h, bh, q0, qb0, lq, kv_len, n_kb, kb_end, nbk, off, qrow, krow, tb;
  bool exists1, causal;
  const uint8_t* bm;
  const uint32_t* bits;  // shared-memory bitmask rows, or null
#ifdef FA_DEBUG_BOUNDS
  int* status;
  long long ext_mask;
#endif

  // last row of Q tile t that exists in the sequence
  __device__ __forceinline__ int last_row(int t) const { return min(q0 + 128 * t + 127, lq - 1); }
  __device__ __forceinline__ bool act_direct(int t, int kb) const {
    if (t == 1 && !exists1) return false;
    if (kb >= n_kb) return false;
    if (causal && kb * 128 > last_row(t) + off) return false;
    if (bm != nullptr && (!FA_IN_BOUNDS(status, static_cast<long long>(qb0 + t) * nbk + kb, 1,
                                        ext_mask) ||
                          bm[static_cast<size_t>(qb0 + t) * nbk + kb] == 0))
      return false;
    return true;
  }
  // kb < kb_end here (every caller walks below kb_end)
  __device__ __forceinline__ bool act(int t, int kb) const {
    if (kBits && bits != nullptr) return t < kRows && ((bits[t * kWpr + (kb >> 5)] >> (kb & 31)) & 1u);
    return act_direct(t, kb);
  }
  // stream (Q tile t, key part hp of kw keys): also skipped when all its keys
  // are past the key length
  __device__ __forceinline__ bool act_s(int t, int hp, int kw, int kb) const {
    return act(t, kb) && kb * 128 + hp * kw < kv_len;
  }
  __device__ __forceinline__ bool any(int kb) const { return act(0, kb) || act(1, kb); }
  __device__ __forceinline__ int next(int kb) const {
    if (kBits && bits != nullptr) {
      while (kb < kb_end) {
        uint32_t x = bits[kb >> 5];
        if (kRows == 2) x |= bits[kWpr + (kb >> 5)];
        x >>= (kb & 31);
        if (x != 0u) return min(kb + __ffs(x) - 1, kb_end);
        kb = (kb | 31) + 1;
      }
      return kb_end;
    }
    while (kb < kb_end && !any(kb)) ++kb;
    return kb;
  }
};

// Barrier `kId` among the 256 threads of the two softmax warpgroups of a Q tile.
template <int kId>
__device__ __forceinline__ void named_bar_sync() {
  asm volatile("bar.sync %0, 256;" ::"n"(kId) : "memory");
}

// POS: the dropout counter is offset by the call's row / key positions in a
// longer sequence (instantiated only with dropout and the direct mask walk; the
// other instances see compile-time zeros).
template <int D, bool DROPOUT, bool BITS, bool POS = false>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, FwdCfg<D>::MIN_BLOCKS)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using L = FwdLayout<D>;
  using C = FwdCfg<D>;
  constexpr int NQ = C::NQ, NS = C::NS, KS = C::KS, KW = C::KW;
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {  // the swizzled layouts need 1024-byte alignment
    if (threadIdx.x == 0 && p.status) atomicExch(p.status, kStatusInternal);
    return;
  }
  auto bar = [&](int i) -> uint32_t { return sbase + L::OFF_BAR + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L::OFF_MISC + 4);
  const WaitGuard g{abort_flag, p.status, p.timeout_ns};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  FwdWork<NQ, L::BIT_WORDS / NQ, BITS> w;
  {
    const int nqp = (p.rows.nq + 128 * NQ - 1) / (128 * NQ);
    int tile = 0;
    grid_unit(blockIdx.x, p.B * p.H, nqp, p.group_heads, &w.bh, &tile);
    const int qp = nqp - 1 - tile;  // heaviest causal rows first
    w.q0 = qp * 128 * NQ;
    w.qb0 = qp * NQ;
    w.b = w.bh / p.H;
    w.h = w.bh % p.H;
    const Seq sq = seq_of(p.rows, w.b);
    // a sequence shorter than the longest has no tile here: leave before any
    // set-up (the whole CTA takes this branch)
    if (w.q0 >= sq.lq) return;
    w.lq = sq.lq;
    w.qrow = sq.q0;
    w.krow = sq.k0;
    w.tb = sq.tb;
    w.off = sq.lk - sq.lq;
    w.exists1 = NQ == 2 && (w.q0 + 128) < sq.lq;
    int kv = sq.lk;
    if (p.seqlens != nullptr && FA_IN_BOUNDS(p.status, w.b, 1, p.ext.seqlens))
      kv = max(0, min(p.seqlens[w.b], sq.lk));
    w.kv_len = kv;
    w.n_kb = (kv + 127) / 128;
    w.causal = p.causal != 0;
    if (w.causal) {
      const int last = w.last_row(w.exists1 ? 1 : 0) + w.off;  // last key any row may see
      w.kb_end = last < 0 ? 0 : min(w.n_kb, last / 128 + 1);
    } else {
      w.kb_end = w.n_kb;
    }
    w.nbk = p.nbk;
    w.bm = p.block_mask;
    w.bits = nullptr;
#ifdef FA_DEBUG_BOUNDS
    w.status = p.status;
    w.ext_mask = p.ext.mask;
#endif
  }
  constexpr int kWpr = L::BIT_WORDS / NQ;
  if (BITS && w.bm != nullptr && (w.kb_end + 31) / 32 <= kWpr) {
    // every thread takes part: a warp's lanes test 32 consecutive K/V tiles
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + L::OFF_BITS);
    const int words = (w.kb_end + 31) / 32;
    for (int t = 0; t < NQ; ++t)
      for (int wi = warp; wi < words; wi += C::THREADS / 32) {
        const int kb = wi * 32 + lane;
        const uint32_t word = __ballot_sync(0xffffffffu, kb < w.kb_end && w.act_direct(t, kb));
        if (lane == 0) bits[t * kWpr + wi] = word;
      }
    w.bits = bits;  // read after the __syncthreads below
  }

  if (threadIdx.x == 0) {
    *abort_flag = 0u;
    for (int t = 0; t < 2; ++t) mbar_init(bar(L::B_QFULL + t), 1);
    for (int s = 0; s < NS * L::S_BUFS; ++s) mbar_init(bar(L::B_SFULL + s), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(L::B_PFULL + s), 4);  // one arrival per softmax warp
      mbar_init(bar(L::B_ODONE + s), 1);
    }
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(bar(L::B_KFULL + s), 1);
      mbar_init(bar(L::B_VFULL + s), 1);
      mbar_init(bar(L::B_KVEMPTY + s), 1);
      if constexpr (L::SPLIT_RELEASE) mbar_init(bar(L::B_VEMPTY + s), 1);
    }
    mbar_init(bar(L::B_DRAIN), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Each role runs inside the branch that sets its register budget, so that
  // the compiler allocates every role's code under its own limit.
  if (warp < 4) {
  if constexpr (C::SPLIT_REGS) setmaxnreg_dec<C::REGS_CTL>();
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      for (int t = 0; t < 2; ++t) {
        if (t == 1 && !w.exists1) break;
        mbar_arrive_expect_tx(bar(L::B_QFULL + t), L::TILE);
        for (int pn = 0; pn < L::PANELS; ++pn)
          tma_load_4d(sbase + L::OFF_Q + t * L::TILE + pn * L::PANEL, &tm_q, bar(L::B_QFULL + t),
                      64 * pn, w.qrow + w.q0 + 128 * t, w.h, w.tb);
      }
      int it = 0;
      for (int kb = w.next(0); kb < w.kb_end; kb = w.next(kb + 1), ++it) {
        const int s = it % L::STAGES;
        const uint32_t ph = (it / L::STAGES) & 1u;
        // the stage's K (SPLIT_RELEASE: V has its own producer) or K and V
        // are free again
        if (it >= L::STAGES && !mbar_wait(bar(L::B_KVEMPTY + s), ph ^ 1u, g)) break;
        const uint32_t kdst = sbase + L::OFF_KV + s * 2 * L::TILE;
        const uint32_t vdst = kdst + L::TILE;
        mbar_arrive_expect_tx(bar(L::B_KFULL + s), L::TILE);
        for (int pn = 0; pn < L::PANELS; ++pn)
          tma_load_4d(kdst + pn * L::PANEL, &tm_k, bar(L::B_KFULL + s), 64 * pn, w.krow + kb * 128,
                      w.h / p.group, w.tb);  // the group's K / V head
        if constexpr (!L::SPLIT_RELEASE) {
          mbar_arrive_expect_tx(bar(L::B_VFULL + s), L::TILE);
          for (int pn = 0; pn < L::PANELS; ++pn)
            tma_load_4d(vdst + pn * L::PANEL, &tm_v, bar(L::B_VFULL + s), 64 * pn,
                        w.krow + kb * 128, w.h / p.group, w.tb);
        }
      }
      if (*abort_flag) {  // let the copies already issued land before the CTA exits
        for (int j = max(0, it - L::STAGES); j < it; ++j) {
          const int s = j % L::STAGES;
          const uint32_t ph = (j / L::STAGES) & 1u;
          mbar_wait_drain(bar(L::B_KFULL + s), ph, 100000000ull);
          if constexpr (!L::SPLIT_RELEASE) mbar_wait_drain(bar(L::B_VFULL + s), ph, 100000000ull);
        }
        mbar_wait_drain(bar(L::B_QFULL + 0), 0, 100000000ull);
        if (w.exists1) mbar_wait_drain(bar(L::B_QFULL + 1), 0, 100000000ull);
      }
    }
  } else if (L::SPLIT_RELEASE && warp == 2) {
    // ------------------------------------------------------------ TMA of V
    // (SPLIT_RELEASE: V tiles have their own producer, so that the next K
    // never waits behind a V that waits for its PV)
    if (lane == 0) {
      tma_prefetch_map(&tm_v);
      int it = 0;
      for (int kb = w.next(0); kb < w.kb_end; kb = w.next(kb + 1), ++it) {
        const int s = it % L::STAGES;
        const uint32_t ph = (it / L::STAGES) & 1u;
        if (it >= L::STAGES && !mbar_wait(bar(L::B_VEMPTY + s), ph ^ 1u, g)) break;
        const uint32_t vdst = sbase + L::OFF_KV + s * 2 * L::TILE + L::TILE;
        mbar_arrive_expect_tx(bar(L::B_VFULL + s), L::TILE);
        for (int pn = 0; pn < L::PANELS; ++pn)
          tma_load_4d(vdst + pn * L::PANEL, &tm_v, bar(L::B_VFULL + s), 64 * pn, w.krow + kb * 128,
                      w.h / p.group, w.tb);
      }
      if (*abort_flag) {
        for (int j = max(0, it - L::STAGES); j < it; ++j)
          mbar_wait_drain(bar(L::B_VFULL + j % L::STAGES), (j / L::STAGES) & 1u, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      // the stream loops unroll while they are short (keeps the issuer's
      // registers in check with four streams)
      constexpr int kUnrollS = KS == 1 ? NS : 1;
      constexpr uint32_t kIdS = idesc_bf16(128, KW, false, false);
      constexpr uint32_t kIdPV = idesc_bf16(128, D, false, true);
      uint32_t q_ready = 0u;  // bit t: Q tile t has landed
      uint32_t o_init = 0u;  // bit s: stream s has accumulated into its O
      uint32_t p_par = 0u;   // bit s: parity of stream s's next P-full phase
      bool ok = true;

      // S of stream s = (Q tile s / KS, key part s % KS) for the K tile at kaddr
      auto issue_s = [&](int s, uint32_t kaddr) {
        const uint32_t qaddr = sbase + L::OFF_Q + (s / KS) * L::TILE;
        const uint32_t kpart = kaddr + static_cast<uint32_t>((s % KS) * KW) * 128u;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::PANEL + (kk & 3) * 32;
          mma_ss(tmem + KW * s, sdesc_sw128(qaddr + off, 16, 1024),
                 sdesc_sw128(kpart + off, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(L::B_SFULL + s));
      };
      auto ensure_q = [&](int t) -> bool {
        if ((q_ready >> t) & 1u) return true;
        if (!mbar_wait(bar(L::B_QFULL + t), 0, g)) return false;
        q_ready |= 1u << t;
        return true;
      };

      if constexpr (L::S_BUFS == 2) {
        // One stream, two S / P buffers: tile n's S goes to buffer n & 1, and
        // S of the tile after next is issued right behind this tile's PV into
        // the buffer that PV has just read, so the tensor pipe computes it
        // while the softmax works on the next tile.  One K / V stage: tile n's
        // K and V are the n-th fills of their barriers (parity n & 1).
        const uint32_t kaddr = sbase + L::OFF_KV, vaddr = kaddr + L::TILE;
        auto issue_s_buf = [&](uint32_t buf) {
          const uint32_t qaddr = sbase + L::OFF_Q;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::PANEL + (kk & 3) * 32;
            mma_ss(tmem + KW * buf, sdesc_sw128(qaddr + off, 16, 1024),
                   sdesc_sw128(kaddr + off, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(L::B_SFULL + buf));
          mma_commit(bar(L::B_KVEMPTY));  // the K tile is free once its S is done
        };
        int kb = w.next(0);
        int kb1 = kb < w.kb_end ? w.next(kb + 1) : w.kb_end;
        if (kb < w.kb_end) {
          ok = mbar_wait(bar(L::B_KFULL), 0, g) && ensure_q(0);
          if (ok) {
            tc_fence_after();
            issue_s_buf(0);
          }
        }
        if (ok && kb1 < w.kb_end) {
          ok = mbar_wait(bar(L::B_KFULL), 1, g);
          if (ok) {
            tc_fence_after();
            issue_s_buf(1);
          }
        }
        for (int it = 0; ok && kb < w.kb_end; ++it) {
          const int kb2 = kb1 < w.kb_end ? w.next(kb1 + 1) : w.kb_end;
          const uint32_t buf = static_cast<uint32_t>(it) & 1u;
          if (!mbar_wait(bar(L::B_VFULL), buf, g) || !mbar_wait(bar(L::B_PFULL), buf, g)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < KW / 16; ++kk)
            mma_ts(tmem + L::O_COL, tmem + KW * buf + 8 * kk,
                   sdesc_sw128(vaddr + kk * 2048, L::PANEL, 1024), kIdPV,
                   (it > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(L::B_ODONE));
          mma_commit(bar(L::B_VEMPTY));  // the V tile is free once its PV is done
          if (kb2 < w.kb_end) {
            if (!mbar_wait(bar(L::B_KFULL), buf, g)) break;  // tile it + 2: parity it & 1
            tc_fence_after();
            issue_s_buf(buf);
          }
          kb = kb1;
          kb1 = kb2;
        }
      } else {
        int kb = w.next(0);
        int it = 0;
        if (kb < w.kb_end) {
          ok = mbar_wait(bar(L::B_KFULL + 0), 0, g);
  #pragma unroll(kUnrollS)
          for (int s = 0; s < NS; ++s) {
            if (!ok || !w.act_s(s / KS, s % KS, KW, kb)) continue;
            ok = ensure_q(s / KS);
            if (ok) {
              tc_fence_after();
              issue_s(s, sbase + L::OFF_KV);
            }
          }
        }
        while (ok && kb < w.kb_end) {
          const int st = it % L::STAGES;
          const uint32_t ph = (it / L::STAGES) & 1u;
          const int kbn = w.next(kb + 1);
          const int sn = (it + 1) % L::STAGES;
          const uint32_t phn = ((it + 1) / L::STAGES) & 1u;
          bool kn_ready = false;
          if (!mbar_wait(bar(L::B_VFULL + st), ph, g)) break;
          const uint32_t vaddr = sbase + L::OFF_KV + st * 2 * L::TILE + L::TILE;
  #pragma unroll(kUnrollS)
          for (int s = 0; s < NS; ++s) {
            if (!ok) break;
            if (w.act_s(s / KS, s % KS, KW, kb)) {
              if (!mbar_wait(bar(L::B_PFULL + s), (p_par >> s) & 1u, g)) {
                ok = false;
                break;
              }
              p_par ^= 1u << s;
              tc_fence_after();
              // this stream's keys are rows [KW (s % KS), KW (s % KS) + KW) of the V tile
              const uint32_t vpart = vaddr + static_cast<uint32_t>((s % KS) * KW) * 128u;
  #pragma unroll
              for (int kk = 0; kk < KW / 16; ++kk)
                mma_ts(tmem + L::O_COL + D * s, tmem + KW * s + 8 * kk,
                       sdesc_sw128(vpart + kk * 2048, L::PANEL, 1024), kIdPV,
                       (((o_init >> s) & 1u) != 0u || kk > 0) ? 1u : 0u);
              o_init |= 1u << s;
              mma_commit(bar(L::B_ODONE + s));
            }
            if (kbn < w.kb_end && w.act_s(s / KS, s % KS, KW, kbn)) {
              if (!kn_ready) {
                if (!mbar_wait(bar(L::B_KFULL + sn), phn, g)) {
                  ok = false;
                  break;
                }
                kn_ready = true;
              }
              if (!ensure_q(s / KS)) {
                ok = false;
                break;
              }
              tc_fence_after();
              issue_s(s, sbase + L::OFF_KV + sn * 2 * L::TILE);
            }
          }
          if (!ok) break;
          mma_commit(bar(L::B_KVEMPTY + st));
          kb = kbn;
          ++it;
        }
      }
      // every MMA issued above has completed once this commit arrives
      mma_commit(bar(L::B_DRAIN));
      mbar_wait_drain(bar(L::B_DRAIN), 0, 1000000000ull);
      for (int t = 0; t < 2; ++t)
        if ((t == 0 || w.exists1) && !((q_ready >> t) & 1u))
          mbar_wait_drain(bar(L::B_QFULL + t), 0, 100000000ull);
    }
  }
  } else {
    if constexpr (C::SPLIT_REGS) setmaxnreg_inc<C::REGS_SOFTMAX>();
    // -------------------------------------------------------------- softmax
    const int s = (warp - 4) >> 2;  // stream
    const int t = s / KS;           // Q tile
    const int hp = s % KS;          // key part
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const int i = w.q0 + 128 * t + r;
    if (t == 0 || w.exists1) {
      const uint32_t lane_addr = tmem + (static_cast<uint32_t>(wq * 32) << 16);
      const uint32_t s_base = lane_addr + KW * s;
      const uint32_t o_addr = lane_addr + L::O_COL + D * s;
      float m = -INFINITY;  // reference maximum, log2 units of scaled scores
      float l = 0.f;        // row sum of exp2(x - m)
      uint32_t cnt = 0;     // active K/V tiles processed so far
      bool ok = true;
      for (int kb = w.next(0); kb < w.kb_end; kb = w.next(kb + 1)) {
        if (!w.act_s(t, hp, KW, kb)) continue;
        // S / P buffer of this tile (tiles alternate when there are two)
        const uint32_t buf = L::S_BUFS == 2 ? (cnt & 1u) : 0u;
        const uint32_t s_addr = s_base + KW * NS * buf;
        const uint32_t s_par = L::S_BUFS == 2 ? ((cnt >> 1) & 1u) : (cnt & 1u);
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_SFULL + s + NS * buf), s_par, g));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[KW];
        tmem_ld32<0>(s_addr + 0, sr);
        tmem_ld32<32>(s_addr + 32, sr);
        if constexpr (KW == 128) {
          tmem_ld32<64>(s_addr + 64, sr);
          tmem_ld32<96>(s_addr + 96, sr);
        }
        tmem_wait_ld32<0>(sr);
        tmem_wait_ld32<32>(sr);
        if constexpr (KW == 128) {
          tmem_wait_ld32<64>(sr);
          tmem_wait_ld32<96>(sr);
        }

        const int j0 = kb * 128 + KW * hp;  // first key of this block
        // masking is needed where a key of this block lies past the first
        // row's causal limit, or past the key length
        const bool need_mask =
            (w.causal && j0 + KW - 1 > w.q0 + 128 * t + w.off) || (j0 + KW > w.kv_len);
        // row maximum with independent partial maxima (short dependency chains;
        // as many as the register budget allows), two scores per max instruction
        constexpr int kParts = C::MAX_PARTS;
        float mxp[kParts];
#pragma unroll
        for (int u = 0; u < kParts; ++u) mxp[u] = -INFINITY;
        if (need_mask) {
          const int lim = w.causal ? min(w.kv_len - j0, i + w.off - j0 + 1) : (w.kv_len - j0);
#pragma unroll
          for (int j = 0; j < KW; ++j)
            if (j >= lim) sr[j] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int c = 0; c < KW / 2; ++c)
          mxp[c % kParts] =
              fmax3(mxp[c % kParts], __uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1]));
        float mx = mxp[0];
#pragma unroll
        for (int u = 1; u < kParts; ++u) mx = fmaxf(mx, mxp[u]);
        mx *= p.scale_log2;
        const float m_new = (mx > m + kRescaleThreshold) ? mx : m;
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = fast_exp2(m - m_use);  // 0 on the first tile, 1 if unchanged
        // scaling and row sum on score pairs (one paired instruction each)
        constexpr int kSums = kParts / 2;
        float2 rsp[kSums];
#pragma unroll
        for (int u = 0; u < kSums; ++u) rsp[u] = make_float2(0.f, 0.f);
        const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 nm2 = make_float2(-m_use, -m_use);
#pragma unroll
        for (int c = 0; c < KW / 2; ++c) {
          const float2 x =
              fma2(make_float2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), sl2, nm2);
          const float2 e = make_float2(fast_exp2(x.x), fast_exp2(x.y));
          rsp[c % kSums] = add2(rsp[c % kSums], e);
          sr[2 * c] = __float_as_uint(e.x);
          sr[2 * c + 1] = __float_as_uint(e.y);
        }
        float rs = 0.f;
#pragma unroll
        for (int u = 0; u < kSums; ++u) rs += rsp[u].x + rsp[u].y;
        l = l * alpha + rs;
        m = m_new;

        uint32_t pk[KW / 2];
        if constexpr (DROPOUT) {
          // Philox call gq of this row covers keys j0 + 8 gq .. j0 + 8 gq + 7;
          // its word u holds the uniforms of keys j0 + 8 gq + 2u (low half) and
          // j0 + 8 gq + 2u + 1 (high half), i.e. exactly bf16 pair 4 gq + u.
          // high half >= t  <=>  word >= t << 16.
          const uint32_t thr = p.drop_threshold;
          const uint32_t thr_hi = thr << 16;
#pragma unroll
          for (int gq = 0; gq < KW / 8; ++gq) {
            const Philox4 rnd = philox4x32_10(
                (POS ? p.drop_kgrp0 : 0u) + static_cast<uint32_t>((j0 >> 3) + gq),
                (POS ? p.drop_row0 : 0u) + static_cast<uint32_t>(i), static_cast<uint32_t>(w.h),
                static_cast<uint32_t>(w.b), p.rk);
            const uint32_t wv[4] = {rnd.w0, rnd.w1, rnd.w2, rnd.w3};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int c = 4 * gq + u;
              const float lo = ((wv[u] & 0xFFFFu) >= thr) ? __uint_as_float(sr[2 * c]) : 0.f;
              const float hi = (wv[u] >= thr_hi) ? __uint_as_float(sr[2 * c + 1]) : 0.f;
              pk[c] = pack_bf16(lo, hi);
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < KW / 2; ++c)
            pk[c] = pack_bf16(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1]));
        }
        tmem_st32<0>(s_addr + 0, pk);
        if constexpr (KW == 128) tmem_st32<32>(s_addr + 32, pk);

        if (cnt > 0) {
          // previous O += P V is complete (it precedes the S MMA just consumed)
          ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_ODONE + s), (cnt - 1) & 1u, g));
          if (!ok) break;
          tc_fence_after();
          if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t orr[32];
              tmem_ld32<0>(o_addr + 32 * c, orr);
              tmem_wait_ld32<0>(orr);
#pragma unroll
              for (int k = 0; k < 16; ++k) {
                const float2 o2 = mul2(make_float2(__uint_as_float(orr[2 * k]), __uint_as_float(orr[2 * k + 1])),
                                       make_float2(alpha, alpha));
                orr[2 * k] = __float_as_uint(o2.x);
                orr[2 * k + 1] = __float_as_uint(o2.y);
              }
              tmem_st32<0>(o_addr + 32 * c, orr);
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::B_PFULL + s));
        ++cnt;
      }

      // ------------------------------------------------------------ epilogue
      if (ok && cnt > 0)
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_ODONE + s), (cnt - 1) & 1u, g));
      const bool row_ok = i < w.lq;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + w.tb * p.so.b +
                            w.h * p.so.h + static_cast<long long>(w.qrow + i) * p.so.r;
      float* lse_out = p.lse + w.tb * p.lse_sb + w.h * p.lse_sh + w.qrow + i;
#ifdef FA_DEBUG_BOUNDS
      const long long o_row = orow - reinterpret_cast<__nv_bfloat16*>(p.o);
      const long long lse_off = lse_out - p.lse;
#endif
      if constexpr (KS == 1) {
        if (ok) {
          tc_fence_after();
          const float inv = (l > 0.f) ? p.drop_rscale / l : 0.f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t orr[32];
            if (cnt > 0) {
              tmem_ld32<0>(o_addr + 32 * c, orr);
              tmem_wait_ld32<0>(orr);
            } else {
#pragma unroll
              for (int k = 0; k < 32; ++k) orr[k] = 0u;
            }
            uint32_t ob[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const float2 o2 = mul2(make_float2(__uint_as_float(orr[2 * k]), __uint_as_float(orr[2 * k + 1])),
                                     make_float2(inv, inv));
              ob[k] = pack_bf16(o2.x, o2.y);
            }
            if (row_ok && 32 * c < p.d_real &&
                FA_IN_BOUNDS(p.status, o_row + 32 * c, 32, p.ext.o)) {
              uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                dst[k] = make_uint4(ob[4 * k], ob[4 * k + 1], ob[4 * k + 2], ob[4 * k + 3]);
            }
          }
          if (row_ok && FA_IN_BOUNDS(p.status, lse_off, 1, p.ext.lse))
            *lse_out = (l > 0.f) ? (m + log2f(l)) * kLn2 : -INFINITY;
        }
      } else {
        // Merge the two streams of this Q tile.  A stream that processed no
        // block never wrote its O accumulator: it zeroes it first.  Both
        // warpgroups publish their row statistics and meet at a named barrier
        // (reached on every path: every wait above is bounded); then each
        // writes D / 2 output columns from both streams' accumulators.
        if (cnt == 0) {
          uint32_t z[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) z[k] = 0u;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) tmem_st32<0>(o_addr + 32 * c, z);
          tmem_wait_st();
        }
        float2* xch = reinterpret_cast<float2*>(smem + L::OFF_XCH);
        xch[s * 128 + r] = make_float2(m, l);
        tc_fence_before();
        if (t == 0) named_bar_sync<1>();
        else named_bar_sync<2>();
        tc_fence_after();
        const float2 st0 = xch[(KS * t) * 128 + r];
        const float2 st1 = xch[(KS * t + 1) * 128 + r];
        if (ok) {
          const float mm = fmaxf(st0.x, st1.x);
          const float mref = (mm == -INFINITY) ? 0.f : mm;
          const float f0 = fast_exp2(st0.x - mref), f1 = fast_exp2(st1.x - mref);
          const float lt = st0.y * f0 + st1.y * f1;
          const float inv = (lt > 0.f) ? p.drop_rscale / lt : 0.f;
          const float2 g0 = make_float2(f0 * inv, f0 * inv), g1 = make_float2(f1 * inv, f1 * inv);
          const uint32_t oc0 = lane_addr + L::O_COL + D * (KS * t) + (D / 2) * hp;
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t a[32], bb[32];
            tmem_ld32<0>(oc0 + 32 * c, a);
            tmem_ld32<0>(oc0 + D + 32 * c, bb);
            tmem_wait_ld32<0>(a);
            tmem_wait_ld32<0>(bb);
            uint32_t ob[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const float2 x0 = make_float2(__uint_as_float(a[2 * k]), __uint_as_float(a[2 * k + 1]));
              const float2 x1 = make_float2(__uint_as_float(bb[2 * k]), __uint_as_float(bb[2 * k + 1]));
              const float2 o2 = fma2(x1, g1, mul2(x0, g0));
              ob[k] = pack_bf16(o2.x, o2.y);
            }
            if (row_ok && (D / 2) * hp + 32 * c < p.d_real &&
                FA_IN_BOUNDS(p.status, o_row + (D / 2) * hp + 32 * c, 32, p.ext.o)) {
              uint4* dst = reinterpret_cast<uint4*>(orow + (D / 2) * hp + 32 * c);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                dst[k] = make_uint4(ob[4 * k], ob[4 * k + 1], ob[4 * k + 2], ob[4 * k + 3]);
            }
          }
          if (row_ok && hp == 0 && FA_IN_BOUNDS(p.status, lse_off, 1, p.ext.lse))
            *lse_out = (lt > 0.f) ? (mref + log2f(lt)) * kLn2 : -INFINITY;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

template <int D, bool DROPOUT, bool BITS, bool POS = false>
cudaError_t launch_fwd_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const FwdParams& p, cudaStream_t stream) {
  using L = FwdLayout<D>;
  using C = FwdCfg<D>;
  auto kern = fwd_kernel<D, DROPOUT, BITS, POS>;
  // The setmaxnreg split is sized for exactly LAUNCH_REGS registers per thread
  // at launch; with any other count an increase could wait forever.  Checked,
  // with the shared-memory attribute set, once per device and context.
  static OncePerContext prepared;
  cudaError_t e = prepared.run([&]() -> cudaError_t {
    if constexpr (C::SPLIT_REGS) {
      cudaFuncAttributes attr{};
      cudaError_t r = cudaFuncGetAttributes(&attr, kern);
      if (r != cudaSuccess) return r;
      if (attr.numRegs != C::LAUNCH_REGS) return cudaErrorInvalidConfiguration;
    }
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(L::SMEM));
  });
  if (e != cudaSuccess) return e;
  const long long ctas =
      static_cast<long long>((p.rows.nq + 128 * C::NQ - 1) / (128 * C::NQ)) * p.B * p.H;
  if (ctas > 0x7FFFFFFFll) return cudaErrorInvalidConfiguration;
  return launch_overlapped(kern, dim3(static_cast<unsigned>(ctas)), dim3(C::THREADS), L::SMEM,
                           stream, tq, tk, tv, p);
}

// A block mask whose rows fit the bitmask (every CTA's K/V tiles are below nbk)
template <int D>
bool uses_bits(const FwdParams& p) {
  return p.block_mask != nullptr && p.mask_bitmap != 0 &&
         (p.nbk + 31) / 32 <= FwdLayout<D>::BIT_WORDS / FwdCfg<D>::NQ;
}

}  // namespace

cudaError_t launch_fwd(int d, bool dropout, const CUtensorMap& tq, const CUtensorMap& tk,
                       const CUtensorMap& tv, const FwdParams& p, cudaStream_t stream) {
  if (dropout && (p.drop_row0 != 0u || p.drop_kgrp0 != 0u)) {  // a block of a longer sequence
    if (d == 64) return launch_fwd_t<64, true, false, true>(tq, tk, tv, p, stream);
    if (d == 128) return launch_fwd_t<128, true, false, true>(tq, tk, tv, p, stream);
    if (d == 256) return launch_fwd_t<256, true, false, true>(tq, tk, tv, p, stream);
    return cudaErrorInvalidValue;
  }
  if (d == 64) {
    if (uses_bits<64>(p))
      return dropout ? launch_fwd_t<64, true, true>(tq, tk, tv, p, stream)
                     : launch_fwd_t<64, false, true>(tq, tk, tv, p, stream);
    return dropout ? launch_fwd_t<64, true, false>(tq, tk, tv, p, stream)
                   : launch_fwd_t<64, false, false>(tq, tk, tv, p, stream);
  }
  if (d == 128) {
    if (uses_bits<128>(p))
      return dropout ? launch_fwd_t<128, true, true>(tq, tk, tv, p, stream)
                     : launch_fwd_t<128, false, true>(tq, tk, tv, p, stream);
    return dropout ? launch_fwd_t<128, true, false>(tq, tk, tv, p, stream)
                   : launch_fwd_t<128, false, false>(tq, tk, tv, p, stream);
  }
  if (d == 256) {
    if (uses_bits<256>(p))
      return dropout ? launch_fwd_t<256, true, true>(tq, tk, tv, p, stream)
                     : launch_fwd_t<256, false, true>(tq, tk, tv, p, stream);
    return dropout ? launch_fwd_t<256, true, false>(tq, tk, tv, p, stream)
                   : launch_fwd_t<256, false, false>(tq, tk, tv, p, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace fa
