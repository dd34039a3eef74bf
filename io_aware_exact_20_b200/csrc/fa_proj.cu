// Fused QKV projection: Y = X W^T + bias, written straight into head-major
// Q, K, V ([B, H, N, d] each), the layout the attention kernels read.
//
// The pages ask for the IO-aware treatment of the layers around attention,
// each of which reads and writes HBM (suanlizi.com FlashAttention summary,
// section IO-感知优化的普遍性 / 子解法2).  The projection in front of attention
// is a dense contraction, so it runs on the tensor cores; what fusion saves
// is the pass that would otherwise reorder its [T, 3, H, d] output into three
// [B, H, N, d] tensors (one read and one write of 6 T H d bytes).
//
// Persistent kernel, one CTA per SM, walking 128-token x 256-column tiles of
// Y (each 32-column chunk lies inside one head of one of Q / K / V, d being 64
// or 128), column tile fastest so that the CTAs running at once share their
// X rows in L2:
//   warp 0      TMA producer: 64-wide K chunks of X (128 rows) and W (256
//               rows), 128-byte swizzle, into a ring of kStages stages that
//               runs on across tiles
//   warp 1      TMEM allocator (2 x 256 columns) and single-thread MMA
//               issuer: tcgen05.mma kind::f16, M = 128, N = 256, both
//               operands K-major, fp32 accumulators alternating between the
//               two TMEM halves
//   warps 4-7   epilogue: thread = token row; TMEM -> + bias -> bf16 ->
//               Q / K / V rows at their head-major addresses, draining one
//               accumulator while the MMA fills the other
// Every wait is bounded (see ptx.cuh).
#include <cuda_bf16.h>

#include "devctx.h"
#include "fa.h"
#include "kernels.h"
#include "ptx.cuh"
#include "tmap.h"

namespace fa {
namespace {

constexpr int kProjThreads = 256;
constexpr int kStages = 4;
constexpr int kBN = 256;                  // output columns per tile
constexpr uint32_t kPanel = 128u * 128u;  // 128 rows x 64 bf16, one 128-byte-swizzled panel
constexpr uint32_t kPanelW = kBN * 128u;  // kBN rows x 64 bf16
constexpr uint32_t kOffX = 0;
constexpr uint32_t kOffW = kStages * kPanel;
constexpr uint32_t kOffBar = kStages * (kPanel + kPanelW);
constexpr int kBarFull = 0, kBarEmpty = kStages;
constexpr int kBarAccFull = 2 * kStages, kBarAccEmpty = 2 * kStages + 2;
constexpr int kBarDrain = 2 * kStages + 4;
constexpr int kNumBars = 2 * kStages + 5;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kProjSmem = kOffMisc + 16;
static_assert(kProjSmem <= 232448, "shared memory budget");

struct ProjParams {
  __nv_bfloat16* oq;            // Q, K, V: bf16 [B, H, N, d]
  __nv_bfloat16* ok;
  __nv_bfloat16* ov;
  const __nv_bfloat16* bias;    // bf16 [3 H d] or null
  int T, N, H, d, ncols, kchunks;
  int col_tiles, tiles;         // column tiles per row tile, all tiles
  int* status;
  uint64_t timeout_ns;
};

__global__ void __launch_bounds__(kProjThreads, 1)
    qkv_proj_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                    const ProjParams p) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0 && p.status) atomicExch(p.status, kStatusInternal);
    return;
  }
  auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc + 4);
  const WaitGuard g{abort_flag, p.status, p.timeout_ns};
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    *abort_flag = 0u;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kBarFull + s), 1);
      mbar_init(bar(kBarEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(kBarAccFull + b), 1);
      mbar_init(bar(kBarAccEmpty + b), 4);  // one arrival per epilogue warp
    }
    mbar_init(bar(kBarDrain), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 2 * kBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      tma_prefetch_map(&tm_x);
      tma_prefetch_map(&tm_w);
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.tiles; tile += gridDim.x) {
        const int n0 = (tile % p.col_tiles) * kBN, t0 = (tile / p.col_tiles) * 128;
        for (int kc = 0; kc < p.kchunks; ++kc, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          if (it >= kStages && !mbar_wait(bar(kBarEmpty + s), ph ^ 1u, g)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(kBarFull + s), kPanel + kPanelW);
          tma_load_2d(sbase + kOffX + s * kPanel, &tm_x, bar(kBarFull + s), 64 * kc, t0);
          tma_load_2d(sbase + kOffW + s * kPanelW, &tm_w, bar(kBarFull + s), 64 * kc, n0);
        }
      }
      if (*abort_flag) {  // let the copies already issued land before the CTA exits
        for (int j = max(0, it - kStages); j < it; ++j)
          mbar_wait_drain(bar(kBarFull + j % kStages), (j / kStages) & 1u, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t kId = idesc_bf16(128, kBN, false, false);
      int it = 0, j = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.tiles; tile += gridDim.x, ++j) {
        const int buf = j & 1;
        // the epilogue has drained this accumulator (two tiles ago)
        if (j >= 2 && !mbar_wait(bar(kBarAccEmpty + buf), ((j >> 1) - 1) & 1u, g)) break;
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(buf * kBN);
        for (int kc = 0; kc < p.kchunks; ++kc, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(bar(kBarFull + s), (it / kStages) & 1u, g)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t xa = sbase + kOffX + s * kPanel, wa = sbase + kOffW + s * kPanelW;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(acc, sdesc_sw128(xa + kk * 32, 16, 1024), sdesc_sw128(wa + kk * 32, 16, 1024),
                   kId, (kc > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(kBarEmpty + s));
        }
        mma_commit(bar(kBarAccFull + buf));
      }
      // every MMA issued above has completed once this commit arrives
      mma_commit(bar(kBarDrain));
      mbar_wait_drain(bar(kBarDrain), 0, 1000000000ull);
    }
  } else if (warp >= 4) {
    // ----------------------------------------------------------- epilogue
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const int hd = p.H * p.d;
    int j = 0;
    for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++j) {
      const int buf = j & 1;
      const int n0 = (tile % p.col_tiles) * kBN, t0 = (tile / p.col_tiles) * 128;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarAccFull + buf), (j >> 1) & 1u, g))) break;
      tc_fence_after();
      const int t = t0 + r;
      const int b = t / p.N, n = t % p.N;
      const uint32_t acc_addr = lane_addr + static_cast<uint32_t>(buf * kBN);
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t acc[32];
        tmem_ld32<0>(acc_addr + 32 * c, acc);
        tmem_wait_ld32<0>(acc);
        if (c == kBN / 32 - 1) {
          // every column of this accumulator is in registers: hand it back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kBarAccEmpty + buf));
        }
        const int col = n0 + 32 * c;
        const bool col_ok = col < p.ncols;  // the last column tile may reach past 3 H d
        float bv[32];
        if (p.bias != nullptr && col_ok) {
          const uint4* bsrc = reinterpret_cast<const uint4*>(p.bias + col);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const uint4 u = bsrc[q4];
            const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(b2[e]);
              bv[8 * q4 + 2 * e] = f.x;
              bv[8 * q4 + 2 * e + 1] = f.y;
            }
          }
        } else {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) bv[jj] = 0.f;
        }
        if (t < p.T && col_ok) {
          const int which = col / hd;
          const int within = col - which * hd;
          const int h = within / p.d, e0 = within - h * p.d;
          __nv_bfloat16* base = which == 0 ? p.oq : (which == 1 ? p.ok : p.ov);
          uint4* dst = reinterpret_cast<uint4*>(
              base + ((static_cast<long long>(b) * p.H + h) * p.N + n) * p.d + e0);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int jj = 8 * q4 + 2 * e;
              w4[e] = pack_bf16(__uint_as_float(acc[jj]) + bv[jj],
                                __uint_as_float(acc[jj + 1]) + bv[jj + 1]);
            }
            dst[q4] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kBN);
  }
}

}  // namespace

cudaError_t launch_qkv_projection(const void* x, const void* w, const void* bias, void* q, void* k,
                                  void* v, int B, int N, int H, int d, int d_model, int* status,
                                  uint64_t timeout_ns, cudaStream_t stream) {
  const long long T = static_cast<long long>(B) * N;
  CUtensorMap tx, tw;
  TmapDesc a = tmap_desc_zero();
  a.base = x;
  a.dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  a.rank = 2;
  a.dims[0] = static_cast<uint64_t>(d_model);
  a.dims[1] = static_cast<uint64_t>(T);
  a.strides[0] = static_cast<uint64_t>(d_model) * 2;
  a.box[0] = 64;
  a.box[1] = 128;
  TmapDesc wd = a;
  wd.base = w;
  wd.dims[1] = static_cast<uint64_t>(3) * H * d;
  wd.box[1] = kBN;  // rows past 3 H d read as zeros
  if (!tmap_cache().encode(a, &tx) || !tmap_cache().encode(wd, &tw)) return cudaErrorInvalidValue;
  ProjParams p;
  p.oq = static_cast<__nv_bfloat16*>(q);
  p.ok = static_cast<__nv_bfloat16*>(k);
  p.ov = static_cast<__nv_bfloat16*>(v);
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.T = static_cast<int>(T);
  p.N = N;
  p.H = H;
  p.d = d;
  p.ncols = 3 * H * d;
  p.kchunks = (d_model + 63) / 64;
  p.col_tiles = (3 * H * d + kBN - 1) / kBN;
  const long long tiles = static_cast<long long>(p.col_tiles) * ((T + 127) / 128);
  if (tiles > 0x7FFFFFFFll) return cudaErrorInvalidValue;
  p.tiles = static_cast<int>(tiles);
  p.status = status;
  p.timeout_ns = timeout_ns;
  static OncePerContext prepared;
  cudaError_t e = prepared.run([]() {
    return cudaFuncSetAttribute(qkv_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kProjSmem));
  });
  if (e != cudaSuccess) return e;
  // one CTA per SM of the current device (a cheap, cached attribute query)
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (sms < 1) return cudaErrorInvalidValue;
  const int grid = p.tiles < sms ? p.tiles : sms;
  return launch_overlapped(qkv_proj_kernel, dim3(static_cast<unsigned>(grid)), dim3(kProjThreads),
                           kProjSmem, stream, tx, tw, p);
}

}  // namespace fa
