// Cached construction of TMA tensor maps (2-D and 3-D) on the host.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace gptq {

// Encodes (or returns from a small per-thread cache) the tensor map of a
// row-major [dim1, dim0] matrix at `ptr` (dim0 contiguous, rows `row_bytes`
// apart) read in boxes of [box1, box0] elements.  Returns false if the driver
// entry point is unavailable or rejects the arguments.
bool tensor_map_2d(CUtensorMap* out, const void* ptr, CUtensorMapDataType dtype, uint64_t dim0,
                   uint64_t dim1, uint64_t row_bytes, uint32_t box0, uint32_t box1,
                   CUtensorMapSwizzle swizzle);

// Same for a 3-D view: dims[0] contiguous, dims[1] and dims[2] `strides[0]`
// and `strides[1]` bytes apart (any order of strides), boxes of box[0..2].
bool tensor_map_3d(CUtensorMap* out, const void* ptr, CUtensorMapDataType dtype,
                   const uint64_t dims[3], const uint64_t strides[2], const uint32_t box[3],
                   CUtensorMapSwizzle swizzle);

}  // namespace gptq
