// Backward pass that allocates nothing: fa_bwd_noalloc.
//
// fa_bwd needs a caller-provided device workspace (dQ accumulators, the
// log2-domain LSE and D_i).  Some callers cannot provide one: code running
// where cudaMalloc is not allowed or not safe to call (inside a custom
// allocator or a memory-pool callback that must not re-enter the allocator,
// plugin hosts that forbid device allocations after start-up, or a framework
// that has pre-reserved all device memory).  For them this file keeps the
// workspace in a fixed, file-scope device array that the CUDA runtime creates
// when it loads this library on a device, and forwards to the normal
// backward with that array as the workspace.
//
// Limits and rules:
//  - the array holds kNoAllocScratchBytes (64 MiB) on every device that loads
//    the library, until the process exits; requests whose workspace
//    (fa_bwd_workspace_size) exceeds it are rejected with FA_ERR_WORKSPACE
//    before anything is launched;
//  - the first call on a device looks up the array's device address with
//    cudaGetSymbolAddress (with that device current) and caches it; make that
//    first call before any stream capture;
//  - every call on a device shares the one array, and it keeps whatever the
//    last call left there; the backward's first launch rewrites every part
//    that must start fresh (it zeroes the dQ accumulators and overwrites the
//    LSE and D rows), so stale contents never leak into a result;
//  - two calls whose kernels overlap on the GPU (different streams, no
//    ordering between them) race on the array and give wrong results:
//    serialise them, for example by issuing them on one stream.
#include <cstdint>
#include <mutex>

#include "fa.h"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t{64} << 20;

static __device__ __align__(256) unsigned char g_bwd_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mutex;

// Device address of g_bwd_scratch on the current device (nullptr on error).
// In host code the array's name is only a host-side handle, never a device
// address, so the address must come from the runtime.
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_bwd_scratch);
    if (e != cudaSuccess || ptr == nullptr) return nullptr;
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" fa_status_t fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                      const float* lse, const void* dout, void* dq, void* dk,
                                      void* dv, int B, int H, int N, int d, float softmax_scale,
                                      int causal, const int32_t* seqlens, float dropout_p,
                                      uint64_t seed, const uint8_t* block_mask, void* stream) {
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (need == 0) return (d != 64 && d != 128) ? FA_ERR_UNSUPPORTED : FA_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return FA_ERR_WORKSPACE;
  void* ws = scratch_address();
  if (ws == nullptr) return FA_ERR_CUDA;
  return fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, softmax_scale, causal, seqlens,
                dropout_p, seed, block_mask, ws, kNoAllocScratchBytes, stream);
}
