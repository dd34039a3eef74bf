// Host-side construction of TMA tensor maps for [B*H, N, d] bf16 tensors.
//
// Each tensor is viewed as 3-D {d, N, B*H} (innermost first) so that a tile
// that runs past row N of one head is zero-filled by the hardware instead of
// reading the next head.  Boxes are 64 elements (128 bytes) wide with the
// 128-byte swizzle; a d = 128 row is fetched as two boxes at x = 0 and x = 64.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

namespace fa {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
  }
  return fn;
}

// bf16 tensor [bh][rows][d] at `base`; box = 64 x box_rows x 1.
// Returns false if the driver rejects the description.
inline bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t d, uint64_t rows,
                           uint64_t bh, uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {d, rows, bh};
  cuuint64_t strides[2] = {d * 2, rows * d * 2};  // bytes, dims 1 and 2
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp32 matrix [rows][cols] at `base`; box = 32 columns (128 bytes) x
// box_rows, 128-byte swizzle.  Used to reduce-add dQ tiles into the backward's
// fp32 accumulators.
inline bool make_tmap_f32_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                             uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {32, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace fa
