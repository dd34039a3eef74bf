// Test-support kernels: the dropout keep bits of every (b, h, i, j), written
// with the same device generator the attention kernels use, and a one-CTA
// wait on a barrier nothing signals, to exercise the bounded-wait path.
#include "kernels.h"
#include "philox.cuh"
#include "ptx.cuh"

namespace fa {
namespace {

__global__ void dropout_mask_kernel(uint8_t* keep, int B, int H, int N, uint32_t threshold,
                                    uint32_t seed_lo, uint32_t seed_hi) {
  const int64_t groups = (N + 7) / 8;
  const int64_t total = static_cast<int64_t>(B) * H * N * groups;
  for (int64_t x = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; x < total;
       x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t g = x % groups;
    const int64_t row = x / groups;  // (b * H + h) * N + i
    const int i = static_cast<int>(row % N);
    const int64_t bh = row / N;
    const int h = static_cast<int>(bh % H);
    const int b = static_cast<int>(bh / H);
    const Philox4 r = philox4x32_10(static_cast<uint32_t>(g), static_cast<uint32_t>(i),
                                    static_cast<uint32_t>(h), static_cast<uint32_t>(b), seed_lo,
                                    seed_hi);
    const uint32_t wv[4] = {r.w0, r.w1, r.w2, r.w3};
    uint8_t* dst = keep + row * N;
    for (int k = 0; k < 8; ++k) {
      const int64_t j = 8 * g + k;
      const uint32_t u = (wv[k >> 1] >> (16 * (k & 1))) & 0xFFFFu;
      if (j < N) dst[j] = u >= threshold ? 1 : 0;
    }
  }
}

__global__ void wait_timeout_kernel(int* status, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar_storage;
  __shared__ uint32_t abort_word;
  const uint32_t bar = smem_u32(&bar_storage);
  if (threadIdx.x == 0) {
    abort_word = 0u;
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitGuard g{&abort_word, status, timeout_ns};
    (void)mbar_wait(bar, 0, g);  // nothing arrives: must give up after timeout_ns
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_dropout_mask(uint8_t* keep, int B, int H, int N, uint32_t threshold,
                                uint32_t seed_lo, uint32_t seed_hi, cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(B) * H * N * ((N + 7) / 8);
  const int threads = 256;
  const int64_t blocks = (total + threads - 1) / threads;
  const int grid = static_cast<int>(blocks < 148 * 64 ? blocks : 148 * 64);
  dropout_mask_kernel<<<grid, threads, 0, stream>>>(keep, B, H, N, threshold, seed_lo, seed_hi);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout_probe(int* status, uint64_t timeout_ns, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace fa
