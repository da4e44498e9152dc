// Cached construction of TMA tensor maps (2-D, row-major) on the host.
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

}  // namespace gptq
