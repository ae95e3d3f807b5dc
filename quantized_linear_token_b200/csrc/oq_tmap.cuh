// TMA tensor maps for the contraction kernels: cuTensorMapEncodeTiled through
// the runtime's driver entry point (no link against the driver library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <string>

#include "oq_internal.h"

namespace oq {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline oq_status tmap_encode_fn(EncodeTiledFn* out) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !f) {
      set_error("cuTensorMapEncodeTiled is not available from the driver");
      return OQ_ERR_CUDA;
    }
    fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  *out = fn;
  return OQ_OK;
}

// A 16-bit K-major operand [rows, K] (rows of K elements, 16-byte aligned),
// fetched in boxes of box_rows x 64 elements with the 128-byte swizzle of
// the tcgen05 operand tiles; rows past the end and columns past K read as 0.
inline oq_status encode_operand_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int64_t rows, int K,
                                    int box_rows, const char* what) {
  EncodeTiledFn fn = nullptr;
  const oq_status st = tmap_encode_fn(&fn);
  if (st != OQ_OK) return st;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error(std::string("cuTensorMapEncodeTiled failed for ") + what + " (code " + std::to_string((int)r) + ")");
    return OQ_ERR_CUDA;
  }
  return OQ_OK;
}

// y [M, N] written by the contraction epilogues in boxes of 32 x 32: fp32 in
// the 128-byte swizzle (128-byte box rows), bf16 in the 64-byte swizzle
// (64-byte box rows); TMA stores clip rows past M
inline oq_status encode_y_map(CUtensorMap* map, void* y, int64_t M, int N, bool bf16 = false) {
  EncodeTiledFn fn = nullptr;
  const oq_status st = tmap_encode_fn(&fn);
  if (st != OQ_OK) return st;
  const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)N * (bf16 ? 2 : 4)};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, y, dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        bf16 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed for y (code " + std::to_string((int)r) + ")");
    return OQ_ERR_CUDA;
  }
  return OQ_OK;
}

}  // namespace oq
