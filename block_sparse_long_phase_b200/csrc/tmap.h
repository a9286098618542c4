// Host-side TMA tensor-map encoding through the driver entry point (no -lcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

namespace star {

inline PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D bf16 tensor [rows][cols] (cols contiguous) read/written in boxes of
// box_rows x box_cols with 128-byte swizzling (box_cols * 2 must be 128).
// Returns false if the driver rejects the map.
inline bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, unsigned long long rows,
                              unsigned long long cols, unsigned box_rows, unsigned box_cols) {
  auto enc = tmap_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [rows][cols] bytes (cols = 64 or 128), box of box_rows whole rows, swizzled
// to match the row length: 128-byte swizzle for 128-byte rows, 64-byte for 64.
inline bool make_tmap_u8_2d(CUtensorMap* map, const void* base, unsigned long long rows,
                            unsigned long long cols, unsigned box_rows) {
  auto enc = tmap_encoder();
  if (!enc || (cols != 64 && cols != 128)) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {(cuuint32_t)cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   cols == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// float32 array of n_quads * 4 elements viewed as [n_quads][4] (16-byte
// rows), boxes of box_quads whole rows; rows past the end read as zero.
inline bool make_tmap_f32_quads(CUtensorMap* map, const float* base, unsigned long long n_quads,
                                unsigned box_quads) {
  auto enc = tmap_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {4, n_quads};
  cuuint64_t strides[1] = {16};
  cuuint32_t bx[2] = {4, box_quads};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, bx,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace star
