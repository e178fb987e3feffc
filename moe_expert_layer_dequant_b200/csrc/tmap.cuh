// Host-side encoding of TMA tensor maps (driver entry point, no -lcuda).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moeffn {

// 2-D tiled map of a row-major [rows][inner] array of `dt` elements whose rows
// are `row_stride_bytes` apart; boxes of [box_rows][box_inner] elements land
// in shared memory row after row. Out-of-range elements read as zero.
cudaError_t encode_tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
                           uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
                           CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_NONE);

}  // namespace moeffn
