// Backward pass that allocates nothing: fa_bwd_noalloc.
//
// fa_bwd needs a caller-provided device workspace (dQ accumulators, the
// log2-domain LSE and D_i).  Some callers cannot provide one: code running
// where cudaMalloc is not allowed or not safe to call (inside a custom
// allocator or a memory-pool callback that must not re-enter the allocator,
// plugin hosts that forbid device allocations after start-up, or a framework
// that has pre-reserved all device memory).  For them this file keeps the
// workspace in a fixed, file-scope device array and forwards to the normal
// backward with that array as the workspace.
//
// Limits and rules:
//  - the array holds kNoAllocScratchBytes (64 MiB) on every device that loads
//    this file's module, until the process exits; requests whose workspace
//    (fa_bwd_workspace_size) exceeds it are rejected with FA_ERR_WORKSPACE
//    before anything is launched;
//  - the array comes into existence when the CUDA runtime loads this file's
//    module on a device.  Under lazy module loading (the default since CUDA
//    12.2) that happens inside the first fa_bwd_noalloc call on the device,
//    when it looks up the array's device address with cudaGetSymbolAddress:
//    that first call is where the 64 MiB is reserved (and where it fails with
//    FA_ERR_CUDA if the device has no room).  Make it at start-up, outside any
//    allocator callback and before any stream capture, or run the process
//    with CUDA_MODULE_LOADING=EAGER so that loading the library reserves it;
//  - the address is cached per device and per context; after a context
//    teardown (cudaDeviceReset) the next call looks it up again;
//  - every call on a device shares the one array, and it keeps whatever the
//    last call left there; the backward's first launch rewrites every part
//    that must start fresh (it zeroes the dQ accumulators and overwrites the
//    LSE and D rows), so stale contents never leak into a result;
//  - two calls whose kernels overlap on the GPU (different streams, no
//    ordering between them) race on the array and give wrong results:
//    serialise them, for example by issuing them on one stream.
#include <cstdint>

#include "devctx.h"
#include "fa.h"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t{64} << 20;

static __device__ __align__(256) unsigned char g_bwd_scratch[kNoAllocScratchBytes];

fa::SymbolAddressCache g_scratch_cache;

// Device address of g_bwd_scratch on the current device (nullptr on error).
// In host code the array's name is only a host-side handle, never a device
// address, so the address must come from the runtime, with the device current.
void* scratch_address() {
  return g_scratch_cache.get([]() -> void* {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_bwd_scratch);
    if (e != cudaSuccess) return nullptr;
    return ptr;
  });
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
