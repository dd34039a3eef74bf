// Host-side construction of TMA tensor maps, with a small cache.
//
// bf16 tensors are viewed as 3-D {d, N, B*H} (innermost first) so that a tile
// that runs past row N of one head is zero-filled by the hardware instead of
// reading the next head.  Boxes are 64 elements (128 bytes) wide with the
// 128-byte swizzle; a d = 128 row is fetched as two boxes at x = 0 and x = 64.
//
// A tensor map only encodes an address, sizes, strides and the box, so an
// encoded map stays valid for as long as the same description is asked for
// again (even if the memory behind the address was freed and reallocated).
// Recently encoded maps are kept, keyed by that whole description, in a
// fixed-size table under a mutex; a hit copies the map out instead of
// encoding it again.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

namespace fa {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
  });
  return fn;
}

// Everything a tensor map encodes (128-byte swizzle, no interleave, 256-byte
// L2 promotion and zero fill are fixed for every map of this library).
struct TmapDesc {
  const void* base;
  uint32_t dtype;  // CUtensorMapDataType
  uint32_t rank;
  uint64_t dims[5];
  uint64_t strides[4];  // bytes, dims 1 .. rank-1
  uint32_t box[5];
};

class TmapCache {
 public:
  bool encode(const TmapDesc& d, CUtensorMap* out) {
    {
      std::lock_guard<std::mutex> lock(mu_);
      for (int i = 0; i < kSlots; ++i)
        if (used_[i] && std::memcmp(&keys_[i], &d, sizeof(TmapDesc)) == 0) {
          *out = maps_[i];
          return true;
        }
    }
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[5], strides[4];
    cuuint32_t box[5], estr[5];
    for (uint32_t i = 0; i < d.rank; ++i) {
      dims[i] = d.dims[i];
      box[i] = d.box[i];
      estr[i] = 1;
      if (i + 1 < d.rank) strides[i] = d.strides[i];
    }
    CUresult r = enc(out, static_cast<CUtensorMapDataType>(d.dtype), d.rank,
                     const_cast<void*>(d.base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    std::lock_guard<std::mutex> lock(mu_);
    keys_[next_] = d;
    maps_[next_] = *out;
    used_[next_] = true;
    next_ = (next_ + 1) % kSlots;
    return true;
  }

 private:
  static constexpr int kSlots = 64;
  std::mutex mu_;
  TmapDesc keys_[kSlots];
  CUtensorMap maps_[kSlots];
  bool used_[kSlots] = {};
  int next_ = 0;
};

inline TmapCache& tmap_cache() {
  static TmapCache cache;
  return cache;
}

inline TmapDesc tmap_desc_zero() {
  TmapDesc d;
  std::memset(&d, 0, sizeof(d));  // padding bytes too: descriptions are compared bytewise
  return d;
}

// bf16 tensor [bh][rows][d] at `base`; box = 64 x box_rows x 1.
// Returns false if the driver rejects the description.
inline bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t d, uint64_t rows,
                           uint64_t bh, uint32_t box_rows) {
  TmapDesc t = tmap_desc_zero();
  t.base = base;
  t.dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  t.rank = 3;
  t.dims[0] = d;
  t.dims[1] = rows;
  t.dims[2] = bh;
  t.strides[0] = d * 2;
  t.strides[1] = rows * d * 2;
  t.box[0] = 64;
  t.box[1] = box_rows;
  t.box[2] = 1;
  return tmap_cache().encode(t, map);
}

// fp32 matrix [rows][cols] at `base`; box = 32 columns (128 bytes) x
// box_rows, 128-byte swizzle.  Used to reduce-add dQ tiles into the backward's
// fp32 accumulators.
inline bool make_tmap_f32_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                             uint32_t box_rows) {
  TmapDesc t = tmap_desc_zero();
  t.base = base;
  t.dtype = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  t.rank = 2;
  t.dims[0] = cols;
  t.dims[1] = rows;
  t.strides[0] = cols * 4;
  t.box[0] = 32;
  t.box[1] = box_rows;
  return tmap_cache().encode(t, map);
}

}  // namespace fa
