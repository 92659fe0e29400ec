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

}  // namespace infini
