// tma_host.h -- host-side construction of TMA tensor maps (cuTensorMapEncodeTiled through the
// runtime's driver entry point, so the library does not link libcuda directly).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace attn {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 4-D map over a row-major [B, S, H, D] tensor: dims (D, H, S, B); a box covers `box_d` head-dim
// elements of one head for `box_rows` consecutive positions. Out-of-range rows read as zero (loads)
// and are skipped (stores / reductions).
inline bool make_map_bshd(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes, int B,
                          int S, int H, int D, int box_d, int box_rows, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(S),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t eb = static_cast<cuuint64_t>(elem_bytes);
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * eb, static_cast<cuuint64_t>(H) * D * eb,
                                 static_cast<cuuint64_t>(S) * H * D * eb};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(box_d), 1, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, dtype, 4, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D map over a packed bf16 [rows, H, D] tensor: dims (D, H, rows); boxes of 64 head-dim elements
// of one head x `box_rows` rows, 128-byte swizzle. `rows` may be a nominal extent: callers must
// only request boxes that lie inside the real tensor.
inline bool make_map_packed_bf16(CUtensorMap* map, const void* base, long long rows, int H, int D, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(H) * D * 2};
  const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 [B, S, H, D] with 128-byte swizzle, boxes of 64 head-dim elements x `rows` positions.
inline bool make_map_bf16_sw128(CUtensorMap* map, const void* base, int B, int S, int H, int D, int rows) {
  return make_map_bshd(map, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, B, S, H, D, 64, rows,
                       CU_TENSOR_MAP_SWIZZLE_128B);
}

// 8-bit [B, S, H, D] (e4m3 codes) with 128-byte swizzle, boxes of 128 head-dim elements x `rows`.
inline bool make_map_u8_sw128(CUtensorMap* map, const void* base, int B, int S, int H, int D, int rows) {
  return make_map_bshd(map, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, S, H, D, 128, rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace attn
