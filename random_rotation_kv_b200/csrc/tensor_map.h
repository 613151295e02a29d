// tensor_map.h — host-side TMA tensor maps (CUtensorMap) over row-major
// [rows][row_elems] arrays, for the batch kernels' tile copies.
//
// Every map here moves raw element bits (unsigned types of the element's
// size) in boxes whose inner extent is exactly 128 bytes, with the 128-byte
// swizzle: inside each 1024-byte shared-memory block, the 16-byte chunk c of
// 128-byte line r sits at chunk position c ^ (r mod 8).  A lane that owns line
// r then reads or writes its chunks without bank conflicts against the 7
// lanes it shares a shared-memory wavefront with.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rrq {

// The driver's cuTensorMapEncodeTiled, looked up once through the runtime
// (no link-time dependency on libcuda); null when unavailable.
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// Map over `rows` rows of `row_elems` elements of `elem_bytes` bytes at
// `base` (16-byte aligned, row pitch a multiple of 16 bytes); boxes of
// 128/elem_bytes elements × `box_rows` rows, 128-byte swizzle, zero fill
// outside the array.  False if the driver rejects the map.
inline bool row_tensor_map(CUtensorMap* map, const void* base, int64_t rows, int row_elems,
                           int elem_bytes, int box_rows) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr || rows <= 0 || rows > (int64_t(1) << 32)) return false;
  const CUtensorMapDataType dt = elem_bytes == 1   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_UINT32;
  const cuuint64_t dims[2] = {cuuint64_t(row_elems), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(row_elems) * cuuint64_t(elem_bytes)};
  const cuuint32_t box[2] = {cuuint32_t(128 / elem_bytes), cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map over `rows` rows of `row_bytes` bytes (a multiple of 16, at most 64) at
// `base`, moved as whole rows in boxes of `box_rows` rows with the 64-byte
// swizzle: inside each 512-byte block of shared memory, the 16-byte chunk c of
// 64-byte line r sits at chunk position c ^ ((r >> 1) mod 4).  Stores clip rows
// past the end of the array.  False if the driver rejects the map.
inline bool code_tensor_map(CUtensorMap* map, const void* base, int64_t rows, int row_bytes,
                            int box_rows) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr || rows <= 0 || rows > (int64_t(1) << 32) || row_bytes % 16 != 0 || row_bytes > 64)
    return false;
  const cuuint64_t dims[2] = {cuuint64_t(row_bytes), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(row_bytes)};
  const cuuint32_t box[2] = {cuuint32_t(row_bytes), cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map over `rows` rows of `row_bytes` bytes (a multiple of 32) at `base`,
// moved in boxes of 32 bytes × `box_rows` rows with the 32-byte swizzle: inside
// each 256-byte block of shared memory, the 16-byte chunk c of 32-byte line r
// sits at chunk position c ^ ((r >> 2) mod 2).  Stores clip rows past the end
// of the array.  False if the driver rejects the map.
inline bool code_box32_tensor_map(CUtensorMap* map, const void* base, int64_t rows, int row_bytes,
                                  int box_rows) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr || rows <= 0 || rows > (int64_t(1) << 32) || row_bytes % 32 != 0) return false;
  const cuuint64_t dims[2] = {cuuint64_t(row_bytes), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(row_bytes)};
  const cuuint32_t box[2] = {32, cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map over `rows` rows of `row_elems` 16-bit elements at `base` (16-byte
// aligned, row pitch a multiple of 16 bytes), moved in boxes of 32 elements
// (64 bytes) × `box_rows` rows with the 64-byte swizzle (as code_tensor_map).
// Stores clip rows past the end of the array.  False if the driver rejects it.
inline bool half_box64_tensor_map(CUtensorMap* map, const void* base, int64_t rows, int row_elems,
                                  int box_rows) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr || rows <= 0 || rows > (int64_t(1) << 32)) return false;
  const cuuint64_t dims[2] = {cuuint64_t(row_elems), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(row_elems) * 2};
  const cuuint32_t box[2] = {32, cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace rrq
