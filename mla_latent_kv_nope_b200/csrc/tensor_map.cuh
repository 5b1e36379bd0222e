// Host-side TMA tensor-map construction for row-major bf16 matrices: the
// driver's cuTensorMapEncodeTiled is looked up once through the runtime (no
// link-time dependency on libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {

using EncodeTiledFnT = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFnT encode_tiled_fn() {
  static EncodeTiledFnT fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFnT>(p);
  }
  return fn;
}

// 16-bit elements (bf16 or fp16: the copy moves bits) [rows, cols] with a
// row pitch of `pitch` elements (pitch * 2 a multiple of 16 bytes), boxes of
// [box_rows, 64] elements (128 bytes), 128-byte swizzle; rows past the end
// read as zeros.
inline bool make_map16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint64_t pitch, uint32_t box_rows) {
  EncodeTiledFnT fn = encode_tiled_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace mla
