// tmap.cuh -- host-side TMA tensor maps (cuTensorMapEncodeTiled, looked up once
// through the runtime's driver entry-point query, so no -lcuda is needed).
#pragma once

#include <stdint.h>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

namespace gdn {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D map over a [rows][cols] row-major region, boxes of [64 rows][128 bytes],
// 128-byte swizzle.
inline bool make_map_rows(CUtensorMap* m, const void* base, CUtensorMapDataType dt,
                          int elem_bytes, uint64_t cols, uint64_t rows) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * elem_bytes};
  const cuuint32_t box[2] = {(cuuint32_t)(128 / elem_bytes), 64};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// 4-D map over a bf16 [B][T][H][128] tensor (coordinates: column, head, time
// step, batch), boxes of 64 columns x 1 head x 64 time steps x 1 batch row,
// 128-byte swizzle; time steps past T read as zeros.
inline bool make_map_bthd(CUtensorMap* m, const void* base, int B, int T, int H) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[3] = {256, (cuuint64_t)H * 256, (cuuint64_t)T * H * 256};
  const cuuint32_t box[4] = {64, 1, 64, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// 4-D map over a [B][T][H][128] tensor of elem_bytes-byte elements (coordinates:
// column, head, time step, batch), boxes of box_cols columns x 1 head x 64 time
// steps x 1 batch row with no swizzle: with box_cols > 128 each time step lands
// as a padded shared-memory row of box_cols elements whose tail columns, like
// time steps past T, read as zeros.
inline bool make_map_bthd_rows(CUtensorMap* m, const void* base, CUtensorMapDataType dt,
                               int elem_bytes, int B, int T, int H, int box_cols) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t row = 128ull * (cuuint64_t)elem_bytes;
  const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[3] = {row, (cuuint64_t)H * row, (cuuint64_t)T * H * row};
  const cuuint32_t box[4] = {(cuuint32_t)box_cols, 1, 64, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, dt, 4, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace gdn
