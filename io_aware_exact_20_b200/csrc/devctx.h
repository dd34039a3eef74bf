// Per-context caching of device addresses of file-scope __device__ variables.
//
// In host code the name of a __device__ variable is only a host-side handle;
// its device address comes from cudaGetSymbolAddress and belongs to the
// context that loaded the module.  After cudaDeviceReset (or any teardown and
// re-creation of the primary context) the module is loaded again, possibly at
// another address, so a cache keyed on the device ordinal alone could hand a
// kernel a stale pointer.  The cache below keys each entry on the ordinal and
// on the unique id of the current context (cuCtxGetId, which never repeats
// within a process) and looks the address up again when the id changes.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

namespace fa {

// Unique id of the calling thread's current context; false if there is none
// or the driver does not provide the id.
inline bool current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Cache of one symbol's device address per (device, context).
class SymbolAddressCache {
 public:
  static constexpr int kMaxDevices = 64;

  // Returns the cached address for the current device and context, or calls
  // `lookup` (which must call cudaGetSymbolAddress with that device current)
  // and caches its result.  nullptr on any failure.
  template <typename Lookup>
  void* get(Lookup lookup) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    unsigned long long ctx = 0;
    std::lock_guard<std::mutex> lock(mu_);
    Entry& e = entries_[dev];
    if (e.ptr != nullptr && current_context_id(&ctx) && e.ctx == ctx) return e.ptr;
    // the lookup also makes the device's context current if it was not yet
    void* ptr = lookup();
    if (ptr == nullptr) return nullptr;
    if (current_context_id(&ctx)) {
      e.ptr = ptr;
      e.ctx = ctx;
    } else {
      e.ptr = nullptr;  // without a context id nothing is cached
    }
    return ptr;
  }

 private:
  struct Entry {
    unsigned long long ctx = 0;
    void* ptr = nullptr;
  };
  std::mutex mu_;
  Entry entries_[kMaxDevices];
};

// Runs a preparation step (function attributes, launch checks) once per
// (device, context): attributes set on a kernel belong to the context that
// loaded its module and are gone after a context teardown.  Two threads may
// both run the step the first time; it must be idempotent.
class OncePerContext {
 public:
  template <typename Prepare>
  cudaError_t run(Prepare prepare) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    unsigned long long ctx = 0;
    const bool have_ctx = current_context_id(&ctx);
    const bool known = dev >= 0 && dev < kMaxDevices;
    if (have_ctx && known && done_[dev].load(std::memory_order_acquire) == ctx + 1)
      return cudaSuccess;
    e = prepare();
    if (e == cudaSuccess && known && current_context_id(&ctx))
      done_[dev].store(ctx + 1, std::memory_order_release);
    return e;
  }

 private:
  static constexpr int kMaxDevices = 64;
  std::atomic<unsigned long long> done_[kMaxDevices] = {};  // context id + 1, 0 = never
};

}  // namespace fa
