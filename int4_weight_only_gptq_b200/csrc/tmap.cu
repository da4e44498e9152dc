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
  int rank, dtype, swizzle;
  uint64_t dim[3], stride[2];
  uint32_t box[3];
  bool operator==(const Key& o) const {
    if (ptr != o.ptr || rank != o.rank || dtype != o.dtype || swizzle != o.swizzle) return false;
    for (int i = 0; i < 3; ++i)
      if (dim[i] != o.dim[i] || box[i] != o.box[i]) return false;
    return stride[0] == o.stride[0] && stride[1] == o.stride[1];
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
  for (int i = 0; i < 3; ++i) {
    h ^= (k.dim[i] + 0x632BE59BD9B4E019ull * (uint64_t)(i + 1)) * 0xC2B2AE3D27D4EB4Full;
    h ^= ((uint64_t)k.box[i] << (8 * i)) * 0x165667B19E3779F9ull;
    h = h ^ (h >> 31);
  }
  h ^= (k.stride[0] * 31 + k.stride[1]) * 0x27D4EB2F165667C5ull;
  h ^= (uint64_t)(k.dtype * 131 + k.swizzle * 7 + k.rank);
  return h ^ (h >> 29);
}

bool encode_cached(CUtensorMap* out, const Key& key) {
  thread_local Entry cache[kSlots];
  Entry& e = cache[hash(key) % kSlots];
  if (e.valid && e.key == key) {
    *out = e.map;
    return true;
  }
  EncodeTiledFn encode = encode_fn();
  if (!encode) return false;
  cuuint64_t gdim[3], gstride[2];
  cuuint32_t box[3], estride[3];
  for (int i = 0; i < key.rank; ++i) {
    gdim[i] = key.dim[i];
    box[i] = key.box[i];
    estride[i] = 1;
  }
  for (int i = 0; i + 1 < key.rank; ++i) gstride[i] = key.stride[i];
  CUtensorMap map;
  if (encode(&map, (CUtensorMapDataType)key.dtype, (cuuint32_t)key.rank, const_cast<void*>(key.ptr),
             gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
             (CUtensorMapSwizzle)key.swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  e.valid = true;
  e.key = key;
  e.map = map;
  *out = map;
  return true;
}

}  // namespace

bool tensor_map_2d(CUtensorMap* out, const void* ptr, CUtensorMapDataType dtype, uint64_t dim0,
                   uint64_t dim1, uint64_t row_bytes, uint32_t box0, uint32_t box1,
                   CUtensorMapSwizzle swizzle) {
  const Key key{ptr, 2, (int)dtype, (int)swizzle, {dim0, dim1, 1}, {row_bytes, 0}, {box0, box1, 1}};
  return encode_cached(out, key);
}

bool tensor_map_3d(CUtensorMap* out, const void* ptr, CUtensorMapDataType dtype,
                   const uint64_t dims[3], const uint64_t strides[2], const uint32_t box[3],
                   CUtensorMapSwizzle swizzle) {
  const Key key{ptr, 3, (int)dtype, (int)swizzle, {dims[0], dims[1], dims[2]},
                {strides[0], strides[1]}, {box[0], box[1], box[2]}};
  return encode_cached(out, key);
}

}  // namespace gptq
