// C ABI of the attention library: argument validation, TMA descriptor set-up
// and kernel launch.  See include/fa.h for the contract of every entry point.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "fa.h"
#include "kernels.h"
#include "tmap.h"

namespace {

// One status word per device, in the library's own device memory (a
// file-scope __device__ variable, so no allocation happens at run time).
__device__ int g_status_word;

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {nullptr};
std::mutex g_status_mutex;
uint64_t g_timeout_ns = 4000000000ull;

int* status_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_status_mutex);
  if (g_status_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(ptr);
  }
  return g_status_ptr[dev];
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Checks shared by the forward and backward entry points.
fa_status_t check_shape(int B, int H, int N, int d, float scale, float dropout_p) {
  if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (!(dropout_p >= 0.f && dropout_p < 1.f)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H > 65535) return FA_ERR_UNSUPPORTED;
  if (N > (1 << 23)) return FA_ERR_UNSUPPORTED;
  // one CTA per (b, h, 128-row tile) in a 1-D grid
  if (static_cast<int64_t>(B) * H * ((N + 127) / 128) > 0x7FFFFFFF) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

bool tensor_ok(const void* p) { return p != nullptr && aligned(p, 16); }

struct Dropout {
  uint32_t threshold;
  float rscale;
};

// Keep test: a 16-bit uniform >= threshold = min(floor(p 2^16), 2^16 - 1);
// kept values are divided by the keep probability 1 - threshold / 2^16.
Dropout dropout_params(float p) {
  const double t = std::floor(static_cast<double>(p) * 65536.0);
  Dropout d;
  d.threshold = t >= 65535.0 ? 65535u : static_cast<uint32_t>(t);
  d.rscale = static_cast<float>(65536.0 / (65536.0 - static_cast<double>(d.threshold)));
  return d;
}

constexpr double kLog2e = 1.4426950408889634074;

int64_t padded_rows(int N) { return (static_cast<int64_t>(N) + 127) / 128 * 128; }

}  // namespace

extern "C" {

const char* fa_status_string(fa_status_t s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "kernel pipeline wait timed out";
    case FA_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

void fa_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns = ns < 1000000ull ? 1000000ull : ns; }

fa_status_t fa_last_device_status(void* stream) {
  int* w = status_word();
  if (w == nullptr) return FA_ERR_CUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return FA_ERR_CUDA;
  if (v == fa::kStatusTimeout) return FA_ERR_TIMEOUT;
  if (v != 0) return FA_ERR_CUDA;
  return FA_OK;
}

fa_status_t fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                   int N, int d, float softmax_scale, int causal, const int32_t* seqlens,
                   float dropout_p, uint64_t seed, const uint8_t* block_mask, void* stream) {
  if (!tensor_ok(q) || !tensor_ok(k) || !tensor_ok(v) || !tensor_ok(o)) return FA_ERR_INVALID_ARG;
  if (lse == nullptr || !aligned(lse, 4)) return FA_ERR_INVALID_ARG;
  if (seqlens != nullptr && !aligned(seqlens, 4)) return FA_ERR_INVALID_ARG;
  fa_status_t st = check_shape(B, H, N, d, softmax_scale, dropout_p);
  if (st != FA_OK) return st;

  int* status = status_word();
  if (status == nullptr) return FA_ERR_CUDA;
  CUtensorMap tq, tk, tv;
  const uint64_t bh = static_cast<uint64_t>(B) * H;
  if (!fa::make_tmap_bf16(&tq, q, d, N, bh, 128) || !fa::make_tmap_bf16(&tk, k, d, N, bh, 128) ||
      !fa::make_tmap_bf16(&tv, v, d, N, bh, 128))
    return FA_ERR_CUDA;

  const Dropout dr = dropout_params(dropout_p);
  fa::FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.seqlens = seqlens;
  p.block_mask = block_mask;
  p.status = status;
  p.B = B;
  p.H = H;
  p.N = N;
  p.nblk = (N + 127) / 128;
  p.scale_log2 = static_cast<float>(static_cast<double>(softmax_scale) * kLog2e);
  p.causal = causal != 0;
  p.group_heads = fa::order_group_heads(B, H, N, d, causal != 0);
  p.drop_threshold = dr.threshold;
  p.drop_rscale = dr.rscale;
  p.seed_lo = static_cast<uint32_t>(seed & 0xFFFFFFFFull);
  p.seed_hi = static_cast<uint32_t>(seed >> 32);
  p.rk = fa::philox_round_keys(seed);
  p.timeout_ns = g_timeout_ns;
  const cudaError_t e =
      fa::launch_fwd(d, dr.threshold != 0, tq, tk, tv, p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128)) return 0;
  const uint64_t rows = static_cast<uint64_t>(B) * H * padded_rows(N);
  const uint64_t bytes = rows * (4ull + 4ull + 4ull * d);
  return static_cast<size_t>((bytes + 255) / 256 * 256);
}

}  // extern "C"

namespace {

// Workspace views and scalar parameters shared by the three backward phases.
fa_status_t bwd_params(fa::BwdParams* p, int B, int H, int N, int d, float softmax_scale,
                       float dropout_p, const void* workspace, size_t workspace_bytes) {
  fa_status_t st = check_shape(B, H, N, d, softmax_scale, dropout_p);
  if (st != FA_OK) return st;
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need)
    return FA_ERR_WORKSPACE;
  int* status = status_word();
  if (status == nullptr) return FA_ERR_CUDA;
  const Dropout dr = dropout_params(dropout_p);
  const int64_t npad = padded_rows(N);
  const uint64_t bh = static_cast<uint64_t>(B) * H;
  *p = fa::BwdParams{};
  p->ws_lse2 = static_cast<float*>(const_cast<void*>(workspace));
  p->ws_delta = p->ws_lse2 + bh * npad;
  p->ws_dq = p->ws_delta + bh * npad;
  p->status = status;
  p->B = B;
  p->H = H;
  p->N = N;
  p->Npad = static_cast<int>(npad);
  p->nblk = (N + 127) / 128;
  p->scale = softmax_scale;
  p->scale_log2 = static_cast<float>(static_cast<double>(softmax_scale) * kLog2e);
  p->drop_threshold = dr.threshold;
  p->drop_rscale = dr.rscale;
  p->timeout_ns = g_timeout_ns;
  return FA_OK;
}

}  // namespace

extern "C" {

fa_status_t fa_bwd_prepare(const void* o, const float* lse, const void* dout, int B, int H, int N,
                           int d, void* workspace, size_t workspace_bytes, void* stream) {
  if (!tensor_ok(o) || !tensor_ok(dout)) return FA_ERR_INVALID_ARG;
  if (lse == nullptr || !aligned(lse, 4)) return FA_ERR_INVALID_ARG;
  fa::BwdParams p;
  // scale and dropout do not enter this phase: validate with neutral values
  fa_status_t st = bwd_params(&p, B, H, N, d, 1.f, 0.f, workspace, workspace_bytes);
  if (st != FA_OK) return st;
  p.o = o;
  p.lse = lse;
  p.dout = dout;
  return fa::launch_bwd_pre(d, p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_OK
                                                                                     : FA_ERR_CUDA;
}

fa_status_t fa_bwd_main(const void* q, const void* k, const void* v, const void* dout, void* dk,
                        void* dv, int B, int H, int N, int d, float softmax_scale, int causal,
                        const int32_t* seqlens, float dropout_p, uint64_t seed,
                        const uint8_t* block_mask, void* workspace, size_t workspace_bytes,
                        void* stream) {
  if (!tensor_ok(q) || !tensor_ok(k) || !tensor_ok(v) || !tensor_ok(dout) || !tensor_ok(dk) ||
      !tensor_ok(dv))
    return FA_ERR_INVALID_ARG;
  if (seqlens != nullptr && !aligned(seqlens, 4)) return FA_ERR_INVALID_ARG;
  fa::BwdParams p;
  fa_status_t st =
      bwd_params(&p, B, H, N, d, softmax_scale, dropout_p, workspace, workspace_bytes);
  if (st != FA_OK) return st;
  CUtensorMap tq, tk, tv, tdo, tdq;
  const uint64_t bh = static_cast<uint64_t>(B) * H;
  if (!fa::make_tmap_bf16(&tq, q, d, N, bh, 128) || !fa::make_tmap_bf16(&tk, k, d, N, bh, 128) ||
      !fa::make_tmap_bf16(&tv, v, d, N, bh, 128) || !fa::make_tmap_bf16(&tdo, dout, d, N, bh, 128) ||
      !fa::make_tmap_f32_2d(&tdq, p.ws_dq, d, bh * static_cast<uint64_t>(p.Npad), 128))
    return FA_ERR_CUDA;
  p.dk = dk;
  p.dv = dv;
  p.seqlens = seqlens;
  p.block_mask = block_mask;
  p.causal = causal != 0;
  p.group_heads = fa::order_group_heads(B, H, N, d, causal != 0);
  p.seed_lo = static_cast<uint32_t>(seed & 0xFFFFFFFFull);
  p.seed_hi = static_cast<uint32_t>(seed >> 32);
  p.rk = fa::philox_round_keys(seed);
  const cudaError_t e = fa::launch_bwd_main(d, p.drop_threshold != 0, tq, tk, tv, tdo, tdq, p,
                                            static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status_t fa_bwd_finish(void* dq, int B, int H, int N, int d, float softmax_scale,
                          const void* workspace, size_t workspace_bytes, void* stream) {
  if (!tensor_ok(dq)) return FA_ERR_INVALID_ARG;
  fa::BwdParams p;
  fa_status_t st = bwd_params(&p, B, H, N, d, softmax_scale, 0.f, workspace, workspace_bytes);
  if (st != FA_OK) return st;
  p.dq = dq;
  return fa::launch_bwd_post(d, p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_OK
                                                                                     : FA_ERR_CUDA;
}

fa_status_t fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dout, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                   float softmax_scale, int causal, const int32_t* seqlens, float dropout_p,
                   uint64_t seed, const uint8_t* block_mask, void* workspace,
                   size_t workspace_bytes, void* stream) {
  // validate everything before the first launch
  if (!tensor_ok(q) || !tensor_ok(k) || !tensor_ok(v) || !tensor_ok(o) || !tensor_ok(dout) ||
      !tensor_ok(dq) || !tensor_ok(dk) || !tensor_ok(dv))
    return FA_ERR_INVALID_ARG;
  if (lse == nullptr || !aligned(lse, 4)) return FA_ERR_INVALID_ARG;
  if (seqlens != nullptr && !aligned(seqlens, 4)) return FA_ERR_INVALID_ARG;
  fa::BwdParams chk;
  fa_status_t st =
      bwd_params(&chk, B, H, N, d, softmax_scale, dropout_p, workspace, workspace_bytes);
  if (st != FA_OK) return st;
  st = fa_bwd_prepare(o, lse, dout, B, H, N, d, workspace, workspace_bytes, stream);
  if (st != FA_OK) return st;
  st = fa_bwd_main(q, k, v, dout, dk, dv, B, H, N, d, softmax_scale, causal, seqlens, dropout_p,
                   seed, block_mask, workspace, workspace_bytes, stream);
  if (st != FA_OK) return st;
  return fa_bwd_finish(dq, B, H, N, d, softmax_scale, workspace, workspace_bytes, stream);
}

fa_status_t fa_debug_dropout_mask(uint8_t* keep, int B, int H, int N, float dropout_p,
                                  uint64_t seed, void* stream) {
  if (keep == nullptr || B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (!(dropout_p >= 0.f && dropout_p < 1.f)) return FA_ERR_INVALID_ARG;
  const Dropout dr = dropout_params(dropout_p);
  const cudaError_t e = fa::launch_dropout_mask(
      keep, B, H, N, dr.threshold, static_cast<uint32_t>(seed & 0xFFFFFFFFull),
      static_cast<uint32_t>(seed >> 32), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status_t fa_debug_wait_timeout(void* stream) {
  int* status = status_word();
  if (status == nullptr) return FA_ERR_CUDA;
  const cudaError_t e =
      fa::launch_wait_timeout_probe(status, g_timeout_ns, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"
