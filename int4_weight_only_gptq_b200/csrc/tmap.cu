// Cached construction of TMA tensor maps.  Encoding is pure host work in the
// driver; a per-thread direct-mapped cache keyed by every argument makes the
// common case (the same weight or activation buffer every call) a copy.
#include <cuda_runtime.h>

#include <mutex>

#include "tmap.h"

namespace gptq {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

struct Key {
  const void* ptr;
  uint64_t dim0, dim1, row_bytes;
  uint32_t box0, box1;
  int dtype, swizzle;
  bool operator==(const Key& o) const {
    return ptr == o.ptr && dim0 == o.dim0 && dim1 == o.dim1 && row_bytes == o.row_bytes &&
           box0 == o.box0 && box1 == o.box1 && dtype == o.dtype && swizzle == o.swizzle;
  }
};

struct Entry {
  bool valid = false;
  Key key;
  CUtensorMap map;
};

constexpr int kSlots = 64;

uint64_t hash(const Key& k) {
  uint64_t h = reinterpret_cast<uint64_t>(k.ptr) * 0x9E3779B97F4A7C15ull;
  h ^= (k.dim0 + 0x632BE59BD9B4E019ull) * 0xC2B2AE3D27D4EB4Full;
  h ^= (k.dim1 + ((uint64_t)k.box0 << 32) + k.box1) * 0x165667B19E3779F9ull;
  h ^= (uint64_t)(k.dtype * 131 + k.swizzle) + k.row_bytes;
  return h ^ (h >> 29);
}

}  // namespace

bool tensor_map_2d(CUtensorMap* out, const void* ptr, CUtensorMapDataType dtype, uint64_t dim0,
                   uint64_t dim1, uint64_t row_bytes, uint32_t box0, uint32_t box1,
                   CUtensorMapSwizzle swizzle) {
  thread_local Entry cache[kSlots];
  const Key key{ptr, dim0, dim1, row_bytes, box0, box1, (int)dtype, (int)swizzle};
  Entry& e = cache[hash(key) % kSlots];
  if (e.valid && e.key == key) {
    *out = e.map;
    return true;
  }
  EncodeTiledFn encode = encode_fn();
  if (!encode) return false;
  const cuuint64_t gdim[2] = {dim0, dim1};
  const cuuint64_t gstride[1] = {row_bytes};
  const cuuint32_t box[2] = {box0, box1};
  const cuuint32_t estride[2] = {1, 1};
  CUtensorMap map;
  if (encode(&map, dtype, 2, const_cast<void*>(ptr), gdim, gstride, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  e.valid = true;
  e.key = key;
  e.map = map;
  *out = map;
  return true;
}

}  // namespace gptq
