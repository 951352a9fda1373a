// tmap.h — host-side TMA tensor-map encoding shared by the library's entry points.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "cp_attn.h"

namespace cpattn {

// ---- TMA tensor maps --------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tensor map over a bf16 view [B, H, L, d] (strides in elements, innermost 1): dimensions
// (d, L, H, B) with 64 x box_rows x 1 x 1 boxes, 128-byte swizzle, zero fill out of bounds.
inline cp_status_t make_map_bhld(CUtensorMap* m, const void* base, int64_t B, int64_t H, int64_t L, int64_t d,
                                 int64_t sB, int64_t sH, int64_t sL, uint32_t box_rows = 128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return CP_ERR_CUDA;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)L, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)(sL * 2), (cuuint64_t)(sH * 2), (cuuint64_t)(sB * 2)};
  cuuint32_t box[4] = {64, box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CP_OK : CP_ERR_CUDA;
}

}  // namespace cpattn
