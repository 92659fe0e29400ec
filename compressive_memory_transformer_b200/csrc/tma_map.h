// tma_map.h — host-side construction of the TMA tensor maps (cuTensorMapEncodeTiled,
// fetched through the runtime's driver entry point so the library does not link
// libcuda directly).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace infini {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D bf16 map over [planes][rows][128]: box = 64 columns x box_rows rows x 1 plane,
// 128-byte swizzle (one box row is exactly one 128-byte swizzle row). Reads past
// the last row of a plane return zeros; stores past it are dropped.
inline bool make_bf16_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t planes,
                          uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {128, rows, planes};
  const cuuint64_t strides[2] = {128 * 2, 128 * 2 * rows};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D bf16 map over d = 128 features x L rows x H heads x B batch rows, element
// (b, h, l, f) at base + b * sb + h * sh + l * sl + f (strides in elements, each a
// multiple of 8, i.e. 16 bytes): [B, H, L, 128] contiguous and [B, L, H, 128] are
// both such maps. Box = 64 features x box_rows rows x one head x one batch row,
// 128-byte swizzle, as make_bf16_map. Rows past L read as zeros; stores there are
// dropped.
inline bool make_bf16_map4(CUtensorMap* m, const void* base, uint64_t L, uint64_t H, uint64_t B,
                           uint64_t sl, uint64_t sh, uint64_t sb, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {128, L, H, B};
  const cuuint64_t strides[3] = {sl * 2, sh * 2, sb * 2};
  const cuuint32_t box[4] = {64, box_rows, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace infini
