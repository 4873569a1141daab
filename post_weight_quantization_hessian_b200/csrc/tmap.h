// Host helper: 2-D bf16 / fp16 TMA tensor maps, 128-byte (or 64-byte)
// swizzle, zero fill out of bounds. cuTensorMapEncodeTiled is fetched through the runtime's driver
// entry point so the library needs no link-time libcuda.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace slim {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Row-major [outer][inner] matrix of 2-byte elements (bf16 or fp16); box =
// box_outer rows x box_inner columns. The base must be 16-byte aligned and
// inner * 2 a multiple of 16 bytes.
inline bool make_tmap_2byte(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                            uint32_t box_outer, bool fp16,
                            CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                           uint32_t box_outer) {
  return make_tmap_2byte(m, base, inner, outer, box_inner, box_outer, false);
}
inline bool make_tmap_f16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                          uint32_t box_outer) {
  return make_tmap_2byte(m, base, inner, outer, box_inner, box_outer, true);
}

// fp16 with 32-column boxes (64 bytes per row) and the 64-byte swizzle.
inline bool make_tmap_f16_sw64(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                               uint32_t box_outer) {
  return make_tmap_2byte(m, base, inner, outer, box_inner, box_outer, true, CU_TENSOR_MAP_SWIZZLE_64B);
}

}  // namespace slim
