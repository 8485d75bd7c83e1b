// kda_tma.h -- host-side construction of TMA tensor maps (2-D tiled,
// 128-byte swizzle) through the driver entry point cuTensorMapEncodeTiled,
// looked up at run time via the runtime API so the library does not link
// libcuda directly.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

namespace kda {

inline PFN_cuTensorMapEncodeTiled_v12000 tma_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// A row-major [rows][cols] matrix with `row_stride_bytes` between rows,
// read or written in boxes of box_rows x box_cols elements with the 128-byte
// swizzle (box_cols * element size must be 128).  Rows beyond `rows` read as
// zero.  Returns false if the driver rejects the description (alignment of
// the base and stride to 16 bytes, sizes).
inline bool make_tma_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, uint32_t elem_bytes,
                        uint64_t cols, uint64_t rows, uint64_t row_stride_bytes, uint32_t box_cols,
                        uint32_t box_rows) {
  auto fn = tma_encode_fn();
  if (fn == nullptr || rows == 0 || cols == 0) return false;
  if (box_cols * elem_bytes != 128u) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace kda
