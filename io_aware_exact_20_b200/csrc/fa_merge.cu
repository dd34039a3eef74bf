// Combining partial attention results, for attention split over key blocks
// that live in different places (context-parallel attention across GPUs, where
// each GPU holds one block of the keys at a time).
//
// A partial result over a key set K_a is (O_a, LSE_a) with O_a the attention
// output normalised over K_a alone and LSE_a = ln sum_{j in K_a} exp(s_j).  For
// disjoint key sets the result over K_a u K_b is
//   LSE = ln(exp(LSE_a) + exp(LSE_b)),
//   O   = exp(LSE_a - LSE) O_a + exp(LSE_b - LSE) O_b,
// the same rescaling the online softmax applies between key blocks inside
// one kernel (the tiling section of the pages: per-block statistics, then a
// rescale of the partial output).  A part with no key (LSE = -inf) leaves the
// other unchanged; two empty parts stay empty (O = 0, LSE = -inf).
//
// Also here: the fp32 accumulation of bf16 gradient parts (dQ, dK, dV summed
// over key / query blocks) and the final fp32 -> bf16 conversions.
#include <cuda_bf16.h>

#include "fa.h"
#include "ptx.cuh"

namespace fa {
namespace {

// G threads per row; the row's d / 8 chunks of 8 columns are dealt out to them
// round-robin (thread `part` takes chunks part, part + G, ...).  G is the
// largest power of two dividing d / 8 (4, 8, 4, 16, 8, 32 for d = 32, 64, 96,
// 128, 192, 256),
// so it divides 32 and a row's threads sit in one warp: the row's two LSEs are
// read once and passed around by shuffles, and the new LSE is written after
// every thread of the row has read the old one.
__global__ void __launch_bounds__(256) merge_kernel(float* o_acc, float* lse_acc,
                                                    const __nv_bfloat16* o_part,
                                                    const float* lse_part, long long rows, int d,
                                                    int G) {
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = tid / G;
  const int part = static_cast<int>(tid % G);
  const bool live = row < rows;
  const int lane = threadIdx.x & 31;
  const int first = lane - part;  // lane of this row's part 0, in this warp
  float la = 0.f, lb = 0.f;
  if (live && part == 0) {
    la = lse_acc[row];
    lb = lse_part[row];
  }
  // every lane of the warp takes part in the shuffles
  la = __shfl_sync(0xffffffffu, la, first);
  lb = __shfl_sync(0xffffffffu, lb, first);
  if (!live) return;
  const float m = fmaxf(la, lb);
  float fa = 0.f, fb = 0.f, lse = -INFINITY;
  if (m != -INFINITY) {
    const float ea = expf(la - m), eb = expf(lb - m);
    const float s = ea + eb;
    fa = ea / s;
    fb = eb / s;
    lse = m + logf(s);
  }
  for (int c = part; c < d / 8; c += G) {
    const long long off = row * d + 8 * c;
    float4* a = reinterpret_cast<float4*>(o_acc + off);
    const uint4 pb = *reinterpret_cast<const uint4*>(o_part + off);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&pb);
    float4 a0 = a[0], a1 = a[1];
    const float2 b0 = __bfloat1622float2(p2[0]), b1 = __bfloat1622float2(p2[1]);
    const float2 b2 = __bfloat1622float2(p2[2]), b3 = __bfloat1622float2(p2[3]);
    // an empty accumulator may hold anything finite; fa = 0 then discards it
    a0 = make_float4(fa * a0.x + fb * b0.x, fa * a0.y + fb * b0.y, fa * a0.z + fb * b1.x,
                     fa * a0.w + fb * b1.y);
    a1 = make_float4(fa * a1.x + fb * b2.x, fa * a1.y + fb * b2.y, fa * a1.z + fb * b3.x,
                     fa * a1.w + fb * b3.y);
    a[0] = a0;
    a[1] = a1;
  }
  if (part == 0) lse_acc[row] = lse;
}

// acc[i] += part[i] (bf16 -> fp32), 8 elements per thread.
__global__ void __launch_bounds__(256) accumulate_kernel(float* acc, const __nv_bfloat16* part,
                                                         long long n8) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= n8) return;
  float4* a = reinterpret_cast<float4*>(acc) + 2 * t;
  const uint4 pb = reinterpret_cast<const uint4*>(part)[t];
  const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&pb);
  const float2 b0 = __bfloat1622float2(p2[0]), b1 = __bfloat1622float2(p2[1]);
  const float2 b2 = __bfloat1622float2(p2[2]), b3 = __bfloat1622float2(p2[3]);
  float4 a0 = a[0], a1 = a[1];
  a[0] = make_float4(a0.x + b0.x, a0.y + b0.y, a0.z + b1.x, a0.w + b1.y);
  a[1] = make_float4(a1.x + b2.x, a1.y + b2.y, a1.z + b3.x, a1.w + b3.y);
}

// out[i] = bf16(in[i]), 8 elements per thread.
__global__ void __launch_bounds__(256) convert_kernel(__nv_bfloat16* out, const float* in,
                                                      long long n8) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= n8) return;
  const float4* a = reinterpret_cast<const float4*>(in) + 2 * t;
  const float4 a0 = a[0], a1 = a[1];
  reinterpret_cast<uint4*>(out)[t] = make_uint4(pack_bf16(a0.x, a0.y), pack_bf16(a0.z, a0.w),
                                                pack_bf16(a1.x, a1.y), pack_bf16(a1.z, a1.w));
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

unsigned blocks_for(long long threads) { return static_cast<unsigned>((threads + 255) / 256); }

}  // namespace
}  // namespace fa

extern "C" {

fa_status_t fa_merge_partial(float* o_acc, float* lse_acc, const void* o_part,
                             const float* lse_part, int64_t rows, int d, void* stream) {
  if (!fa::aligned16(o_acc) || !fa::aligned16(o_part) || lse_acc == nullptr ||
      lse_part == nullptr || rows < 0)
    return FA_ERR_INVALID_ARG;
  if (d != 32 && d != 64 && d != 96 && d != 128 && d != 192 && d != 256) return FA_ERR_UNSUPPORTED;
  if (rows == 0) return FA_OK;
  const int G = (d / 8) & -(d / 8);  // largest power of two dividing d / 8
  if (rows * G / 256 >= 0x7FFFFFFFll) return FA_ERR_UNSUPPORTED;
  fa::merge_kernel<<<fa::blocks_for(rows * G), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      o_acc, lse_acc, static_cast<const __nv_bfloat16*>(o_part), lse_part, rows, d, G);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status_t fa_accumulate_bf16(float* acc, const void* part, int64_t n, void* stream) {
  if (!fa::aligned16(acc) || !fa::aligned16(part) || n < 0 || n % 8) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (n / 8 / 256 >= 0x7FFFFFFFll) return FA_ERR_UNSUPPORTED;
  fa::accumulate_kernel<<<fa::blocks_for(n / 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      acc, static_cast<const __nv_bfloat16*>(part), n / 8);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status_t fa_convert_f32_bf16(void* out, const float* in, int64_t n, void* stream) {
  if (!fa::aligned16(out) || !fa::aligned16(in) || n < 0 || n % 8) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (n / 8 / 256 >= 0x7FFFFFFFll) return FA_ERR_UNSUPPORTED;
  fa::convert_kernel<<<fa::blocks_for(n / 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<__nv_bfloat16*>(out), in, n / 8);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"
