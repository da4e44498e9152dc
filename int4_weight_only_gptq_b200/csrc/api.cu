// C ABI of the W4A16 GPTQ library: argument checks (fail-closed, before any
// launch), the shape-driven dispatcher, and the per-device state.
//
// The checks restate the runtime contract of the GPTQ-Pro README ("Runtime
// contract": group sizes -1/16/32/64/128/256/512/1024, input features
// divisible by 16, output features divisible by 8; unsupported combinations
// are rejected, never silently routed elsewhere).
#include <cuda_runtime.h>

#include <mutex>

#include "gptq_w4a16.h"
#include "kernels.h"

namespace gptq {
namespace {

// One error word per device, written only by kernels that give up a wait.
__device__ int g_error_word;

// The T buffer of gptq_w4a16_gemm_lora_noalloc: static device memory of the
// library, one per device, shared by every such call on that device.
__device__ __align__(256) uint16_t g_lora_scratch[GPTQ_LORA_SCRATCH_BYTES / 2];

// Hand-over flags of adapters computed inside the layer's launch: slot
// (call number % kTFlagSlots) counts the T CTAs done (low half) and the layer
// CTAs past their wait (high half); the last of those clears it.
__device__ unsigned long long g_t_flags[kTFlagSlots];

constexpr int kMaxDevices = 64;
std::once_flag g_dev_once[kMaxDevices];
DeviceInfo g_dev[kMaxDevices];
int g_dev_status[kMaxDevices];

int query_device(const DeviceInfo** out) {
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) {
    cudaGetLastError();
    return GPTQ_ERR_DEVICE;
  }
  std::call_once(g_dev_once[d], [d] {
    DeviceInfo info;
    info.device = d;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, d) != cudaSuccess) {
      cudaGetLastError();
      g_dev_status[d] = GPTQ_ERR_DEVICE;
      return;
    }
    info.num_sms = prop.multiProcessorCount;
    info.cc_major = prop.major;
    info.cc_minor = prop.minor;
    info.smem_optin = (int)prop.sharedMemPerBlockOptin;
    info.l2_bytes = prop.l2CacheSize;
    if (info.cc_major != 10 || info.cc_minor != 0) {
      g_dev_status[d] = GPTQ_ERR_DEVICE;
      return;
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) {
      cudaGetLastError();
      g_dev_status[d] = GPTQ_ERR_DEVICE;
      return;
    }
    info.error_word = static_cast<int*>(p);
    void* q = nullptr;
    if (cudaGetSymbolAddress(&q, g_lora_scratch) != cudaSuccess) {
      cudaGetLastError();
      g_dev_status[d] = GPTQ_ERR_DEVICE;
      return;
    }
    info.lora_scratch = static_cast<uint16_t*>(q);
    void* f = nullptr;
    if (cudaGetSymbolAddress(&f, g_t_flags) != cudaSuccess) {
      cudaGetLastError();
      g_dev_status[d] = GPTQ_ERR_DEVICE;
      return;
    }
    info.t_flags = static_cast<unsigned long long*>(f);
    g_dev[d] = info;
    g_dev_status[d] = GPTQ_OK;
  });
  if (g_dev_status[d] != GPTQ_OK) return g_dev_status[d];
  *out = &g_dev[d];
  return GPTQ_OK;
}

bool valid_group(int32_t g) {
  switch (g) {
    case -1: case 16: case 32: case 64: case 128: case 256: case 512: case 1024:
      return true;
    default:
      return false;
  }
}

int check_shape(int64_t M, int64_t K, int64_t N, int32_t group) {
  if (M < 0 || K <= 0 || N <= 0) return GPTQ_ERR_SHAPE;
  if (K % 16 != 0 || N % 8 != 0) return GPTQ_ERR_SHAPE;
  if (K > GPTQ_MAX_K || N > GPTQ_MAX_N || M > GPTQ_MAX_M) return GPTQ_ERR_SHAPE;
  if (!valid_group(group)) return GPTQ_ERR_GROUP;
  return GPTQ_OK;
}

int64_t num_groups(int64_t K, int32_t group) {
  if (group == -1 || group >= K) return 1;
  return (K + group - 1) / group;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, int64_t abytes, const void* b, int64_t bbytes) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + (uintptr_t)bbytes && b0 < a0 + (uintptr_t)abytes;
}

int select_kernel(int64_t M, int64_t K, int64_t N, const DeviceInfo& dev, int32_t* split) {
  if (M <= GPTQ_DECODE_MAX_M) {
    if (split) *split = decode_pick_splits(M, K, N, false, dev);
    return GPTQ_KERNEL_DECODE;
  }
  if (split) *split = 1;
  return GPTQ_KERNEL_PREFILL;
}

int gemm_impl(const uint16_t* x, const int32_t* qweight, const uint16_t* scales, int64_t M,
              int64_t K, int64_t N, int32_t group, uint16_t* y, void* stream, int32_t kernel_id,
              int32_t splits) {
  int st = check_shape(M, K, N, group);
  if (st != GPTQ_OK) return st;
  if (kernel_id < GPTQ_KERNEL_AUTO || kernel_id > GPTQ_KERNEL_PREFILL) return GPTQ_ERR_KERNEL;
  if (kernel_id == GPTQ_KERNEL_DECODE && M > GPTQ_DECODE_MAX_M) return GPTQ_ERR_KERNEL;
  if (splits < 0 || splits > 8) return GPTQ_ERR_KERNEL;
  if (!qweight || !scales) return GPTQ_ERR_NULL;
  if (M == 0) return GPTQ_OK;
  if (!x || !y) return GPTQ_ERR_NULL;
  if (!aligned16(x) || !aligned16(qweight) || !aligned16(scales) || !aligned16(y))
    return GPTQ_ERR_ALIGN;
  const int64_t ybytes = M * N * 2;
  if (overlaps(y, ybytes, x, M * K * 2) || overlaps(y, ybytes, qweight, K / 8 * N * 4) ||
      overlaps(y, ybytes, scales, num_groups(K, group) * N * 2))
    return GPTQ_ERR_ALIAS;
  const DeviceInfo* dev = nullptr;
  st = query_device(&dev);
  if (st != GPTQ_OK) return st;
  if (kernel_id == GPTQ_KERNEL_AUTO) kernel_id = select_kernel(M, K, N, *dev, nullptr);
  const int gs = group_shift_of(group);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (kernel_id == GPTQ_KERNEL_DECODE)
    e = launch_decode(x, qweight, scales, y, M, K, N, gs, splits, s, *dev);
  else
    e = launch_prefill(x, qweight, scales, y, M, K, N, gs, s, *dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  return GPTQ_OK;
}

// The adapter path.  t_work: caller-owned T buffer, or (static_t) the
// library's static one.
int lora_impl(const uint16_t* x, const int32_t* qweight, const uint16_t* scales, int64_t M,
              int64_t K, int64_t N, int32_t group, const uint16_t* lora_a,
              const uint16_t* lora_b, int64_t rank, uint16_t* t_work, bool static_t, uint16_t* y,
              void* stream) {
  int st = check_shape(M, K, N, group);
  if (st != GPTQ_OK) return st;
  if (rank < 16 || rank > GPTQ_MAX_LORA_RANK || rank % 16 != 0) return GPTQ_ERR_SHAPE;
  if (static_t && M * rank * 2 > (int64_t)GPTQ_LORA_SCRATCH_BYTES) return GPTQ_ERR_SHAPE;
  if (!qweight || !scales || !lora_a || !lora_b) return GPTQ_ERR_NULL;
  if (M == 0) return GPTQ_OK;
  if (!x || !y || (!static_t && !t_work)) return GPTQ_ERR_NULL;
  if (!aligned16(x) || !aligned16(qweight) || !aligned16(scales) || !aligned16(y) ||
      !aligned16(lora_a) || !aligned16(lora_b) || (!static_t && !aligned16(t_work)))
    return GPTQ_ERR_ALIGN;
  const int64_t xb = M * K * 2, qb = K / 8 * N * 4, sb = num_groups(K, group) * N * 2;
  const int64_t ab = rank * K * 2, bb = N * rank * 2, tb = M * rank * 2, yb = M * N * 2;
  // y and t_work are written: neither may overlap anything else (the static
  // buffer overlaps no caller buffer)
  if (overlaps(y, yb, x, xb) || overlaps(y, yb, qweight, qb) || overlaps(y, yb, scales, sb) ||
      overlaps(y, yb, lora_a, ab) || overlaps(y, yb, lora_b, bb))
    return GPTQ_ERR_ALIAS;
  if (!static_t &&
      (overlaps(y, yb, t_work, tb) || overlaps(t_work, tb, x, xb) ||
       overlaps(t_work, tb, qweight, qb) || overlaps(t_work, tb, scales, sb) ||
       overlaps(t_work, tb, lora_a, ab) || overlaps(t_work, tb, lora_b, bb)))
    return GPTQ_ERR_ALIAS;
  const DeviceInfo* dev = nullptr;
  st = query_device(&dev);
  if (st != GPTQ_OK) return st;
  if (static_t) t_work = dev->lora_scratch;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // up to GPTQ_LORA_DECODE_MAX_M tokens, when the decode launch leaves SMs
  // free: T on CTAs of the layer's own launch, handed over through a flag
  if (M <= GPTQ_LORA_DECODE_MAX_M && decode_lora_fused_fits(M, K, N, rank, *dev)) {
    const cudaError_t e = launch_decode_lora_fused(x, qweight, scales, y, M, K, N,
                                                   group_shift_of(group), t_work, lora_a, lora_b,
                                                   rank, s, *dev);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return GPTQ_ERR_CUDA;
    }
    return GPTQ_OK;
  }
  // up to GPTQ_LORA_DECODE_MAX_M tokens the layer runs on the decode kernel,
  // one CTA per SM: the T launch may use the SMs it leaves free
  int free_sms = 0;
  if (M <= GPTQ_LORA_DECODE_MAX_M) {
    const int64_t ctas = decode_ctas(M, K, N, true, *dev);
    free_sms = ctas < dev->num_sms ? (int)(dev->num_sms - ctas) : 0;
  }
  cudaError_t e = launch_lora_down(x, lora_a, t_work, M, K, rank, free_sms, s, *dev);
  if (e == cudaSuccess)
    e = M <= GPTQ_LORA_DECODE_MAX_M
            ? launch_decode_lora(x, qweight, scales, y, M, K, N, group_shift_of(group), t_work,
                                 lora_b, rank, s, *dev)
            : launch_prefill_pair_lora(x, qweight, scales, y, M, K, N, group_shift_of(group),
                                       t_work, lora_b, rank, s, *dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  return GPTQ_OK;
}

}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" {

int gptq_w4a16_gemm(const uint16_t* x, const int32_t* qweight, const uint16_t* scales, int64_t M,
                    int64_t K, int64_t N, int32_t group, uint16_t* y, void* stream) {
  return gemm_impl(x, qweight, scales, M, K, N, group, y, stream, GPTQ_KERNEL_AUTO, 0);
}

int gptq_w4a16_gemm_kernel(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                           int64_t M, int64_t K, int64_t N, int32_t group, uint16_t* y,
                           void* stream, int32_t kernel_id) {
  return gemm_impl(x, qweight, scales, M, K, N, group, y, stream, kernel_id, 0);
}

int gptq_w4a16_gemm_decode_splits(const uint16_t* x, const int32_t* qweight,
                                  const uint16_t* scales, int64_t M, int64_t K, int64_t N,
                                  int32_t group, uint16_t* y, void* stream, int32_t splits) {
  if (splits < 1) return GPTQ_ERR_KERNEL;
  return gemm_impl(x, qweight, scales, M, K, N, group, y, stream, GPTQ_KERNEL_DECODE, splits);
}

int gptq_w4a16_gemm_grouped(const uint16_t* x, const int32_t* const* qweights,
                            const uint16_t* const* scales, const int64_t* Ns, int32_t count,
                            int64_t M, int64_t K, int32_t group, uint16_t* const* ys,
                            void* stream) {
  if (count < 1 || count > GPTQ_MAX_GROUPED) return GPTQ_ERR_SHAPE;
  if (!qweights || !scales || !Ns || !ys) return GPTQ_ERR_NULL;
  for (int i = 0; i < count; ++i) {
    const int st = check_shape(M, K, Ns[i], group);
    if (st != GPTQ_OK) return st;
  }
  for (int i = 0; i < count; ++i)
    if (!qweights[i] || !scales[i]) return GPTQ_ERR_NULL;
  if (M == 0) return GPTQ_OK;
  if (!x) return GPTQ_ERR_NULL;
  for (int i = 0; i < count; ++i)
    if (!ys[i]) return GPTQ_ERR_NULL;
  if (!aligned16(x)) return GPTQ_ERR_ALIGN;
  for (int i = 0; i < count; ++i)
    if (!aligned16(qweights[i]) || !aligned16(scales[i]) || !aligned16(ys[i]))
      return GPTQ_ERR_ALIGN;
  const int64_t ng = num_groups(K, group);
  for (int i = 0; i < count; ++i) {
    const int64_t ybytes = M * Ns[i] * 2;
    if (overlaps(ys[i], ybytes, x, M * K * 2)) return GPTQ_ERR_ALIAS;
    for (int j = 0; j < count; ++j) {
      if (overlaps(ys[i], ybytes, qweights[j], K / 8 * Ns[j] * 4) ||
          overlaps(ys[i], ybytes, scales[j], ng * Ns[j] * 2) ||
          (j != i && overlaps(ys[i], ybytes, ys[j], M * Ns[j] * 2)))
        return GPTQ_ERR_ALIAS;
    }
  }
  const DeviceInfo* dev = nullptr;
  const int st = query_device(&dev);
  if (st != GPTQ_OK) return st;
  const int gs = group_shift_of(group);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (M <= GPTQ_DECODE_MAX_M) {
    e = launch_decode_grouped(x, qweights, scales, Ns, ys, count, M, K, gs, s, *dev);
  } else {
    for (int i = 0; i < count && e == cudaSuccess; ++i)
      e = launch_prefill(x, qweights[i], scales[i], ys[i], M, K, Ns[i], gs, s, *dev);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  return GPTQ_OK;
}

int gptq_w4a16_gemm_gidx(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                         const int32_t* g_idx, int64_t M, int64_t K, int64_t N, int64_t n_groups,
                         uint16_t* y, void* stream) {
  int st = check_shape(M, K, N, -1);
  if (st != GPTQ_OK) return st;
  if (n_groups < 1 || n_groups > GPTQ_GIDX_MAX_GROUPS) return GPTQ_ERR_SHAPE;
  if (!qweight || !scales || !g_idx) return GPTQ_ERR_NULL;
  if (M == 0) return GPTQ_OK;
  if (!x || !y) return GPTQ_ERR_NULL;
  if (!aligned16(x) || !aligned16(qweight) || !aligned16(scales) || !aligned16(g_idx) ||
      !aligned16(y))
    return GPTQ_ERR_ALIGN;
  const int64_t yb = M * N * 2;
  if (overlaps(y, yb, x, M * K * 2) || overlaps(y, yb, qweight, K / 8 * N * 4) ||
      overlaps(y, yb, scales, n_groups * N * 2) || overlaps(y, yb, g_idx, K * 4))
    return GPTQ_ERR_ALIAS;
  const DeviceInfo* dev = nullptr;
  st = query_device(&dev);
  if (st != GPTQ_OK) return st;
  const cudaError_t e = launch_decode_gidx(x, qweight, scales, g_idx, y, M, K, N, n_groups,
                                           static_cast<cudaStream_t>(stream), *dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  return GPTQ_OK;
}

int gptq_w4a16_gemm_asym(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                         const int32_t* qzeros, int64_t M, int64_t K, int64_t N, int32_t group,
                         uint16_t* y, void* stream) {
  int st = check_shape(M, K, N, group);
  if (st != GPTQ_OK) return st;
  if (N % 32 != 0) return GPTQ_ERR_SHAPE;
  if (!qweight || !scales || !qzeros) return GPTQ_ERR_NULL;
  if (M == 0) return GPTQ_OK;
  if (!x || !y) return GPTQ_ERR_NULL;
  if (!aligned16(x) || !aligned16(qweight) || !aligned16(scales) || !aligned16(qzeros) ||
      !aligned16(y))
    return GPTQ_ERR_ALIGN;
  const int64_t ng = num_groups(K, group), yb = M * N * 2;
  if (overlaps(y, yb, x, M * K * 2) || overlaps(y, yb, qweight, K / 8 * N * 4) ||
      overlaps(y, yb, scales, ng * N * 2) || overlaps(y, yb, qzeros, ng * (N / 8) * 4))
    return GPTQ_ERR_ALIAS;
  const DeviceInfo* dev = nullptr;
  st = query_device(&dev);
  if (st != GPTQ_OK) return st;
  const int gs = group_shift_of(group);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e = M <= GPTQ_DECODE_MAX_M
                            ? launch_decode_asym(x, qweight, scales, qzeros, y, M, K, N, gs, s,
                                                 *dev)
                            : launch_prefill_pair_asym(x, qweight, scales, qzeros, y, M, K, N, gs,
                                                       s, *dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  return GPTQ_OK;
}

int gptq_w4a16_gemm_lora(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                         int64_t M, int64_t K, int64_t N, int32_t group, const uint16_t* lora_a,
                         const uint16_t* lora_b, int64_t rank, uint16_t* t_work, uint16_t* y,
                         void* stream) {
  return lora_impl(x, qweight, scales, M, K, N, group, lora_a, lora_b, rank, t_work, false, y,
                   stream);
}

int gptq_w4a16_gemm_lora_noalloc(const uint16_t* x, const int32_t* qweight,
                                 const uint16_t* scales, int64_t M, int64_t K, int64_t N,
                                 int32_t group, const uint16_t* lora_a, const uint16_t* lora_b,
                                 int64_t rank, uint16_t* y, void* stream) {
  return lora_impl(x, qweight, scales, M, K, N, group, lora_a, lora_b, rank, nullptr, true, y,
                   stream);
}


int gptq_dequant(const int32_t* qweight, const uint16_t* scales, int64_t K, int64_t N,
                 int32_t group, uint16_t* w_out, void* stream) {
  int st = check_shape(0, K, N, group);
  if (st != GPTQ_OK) return st;
  if (!qweight || !scales || !w_out) return GPTQ_ERR_NULL;
  if (!aligned16(qweight) || !aligned16(scales) || !aligned16(w_out)) return GPTQ_ERR_ALIGN;
  const int64_t wbytes = K * N * 2;
  if (overlaps(w_out, wbytes, qweight, K / 8 * N * 4) ||
      overlaps(w_out, wbytes, scales, num_groups(K, group) * N * 2))
    return GPTQ_ERR_ALIAS;
  const DeviceInfo* dev = nullptr;
  st = query_device(&dev);
  if (st != GPTQ_OK) return st;
  cudaError_t e = launch_dequant(qweight, scales, K, N, group_shift_of(group), w_out,
                                 static_cast<cudaStream_t>(stream), *dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  return GPTQ_OK;
}

int gptq_w4a16_select(int64_t M, int64_t K, int64_t N, int32_t group, int32_t* kernel_id,
                      int32_t* split_k) {
  int st = check_shape(M, K, N, group);
  if (st != GPTQ_OK) return st;
  const DeviceInfo* dev = nullptr;
  st = query_device(&dev);
  if (st != GPTQ_OK) return st;
  int32_t split = 1;
  const int k = select_kernel(M, K, N, *dev, &split);
  if (kernel_id) *kernel_id = k;
  if (split_k) *split_k = split;
  return GPTQ_OK;
}

const char* gptq_status_string(int status) {
  switch (status) {
    case GPTQ_OK: return "ok";
    case GPTQ_ERR_NULL: return "null pointer";
    case GPTQ_ERR_SHAPE: return "invalid shape (need M >= 0, K > 0 and K % 16 == 0, N > 0 and N % 8 == 0, within the size limits)";
    case GPTQ_ERR_GROUP: return "unsupported group size (need -1, 16, 32, 64, 128, 256, 512 or 1024)";
    case GPTQ_ERR_ALIGN: return "pointer not 16-byte aligned";
    case GPTQ_ERR_DEVICE: return "no current CUDA device of compute capability 10.0";
    case GPTQ_ERR_CUDA: return "CUDA launch error";
    case GPTQ_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
    case GPTQ_ERR_ALIAS: return "output overlaps an input";
    case GPTQ_ERR_KERNEL: return "kernel id or split count not valid for this call";
    case GPTQ_ERR_INDEX: return "a g_idx entry outside 0 .. n_groups - 1";
    default: return "unknown status";
  }
}

int gptq_device_error(void) {
  const DeviceInfo* dev = nullptr;
  int st = query_device(&dev);
  if (st != GPTQ_OK) return st;
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  int v = 0;
  const int zero = 0;
  if (cudaMemcpy(&v, dev->error_word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(dev->error_word, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  // a kernel that gave up may have left an adapter hand-over slot uncleared
  if (v != 0 && cudaMemset(dev->t_flags, 0, sizeof(unsigned long long) * kTFlagSlots) !=
                    cudaSuccess) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  return v;
}

const char* gptq_version(void) { return "0.1.0"; }

}  // extern "C"
