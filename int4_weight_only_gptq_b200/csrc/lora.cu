// The LoRA adapter's down-projection: T[M, r] = fp16(X[M, K] . lora_a[r, K]^T).
//
// GPTQ-Pro README, "Runtime contract": adapters are LoRA on the linear path;
// the adapter's own output is FP16 (its dtype), summed here in FP32.  T then
// enters the decode kernel (up to 32 tokens) or the prefill pair kernel as
// extra K of the layer's product, where T . lora_b^T is added to the FP32
// accumulator.
//
// Deterministic forms (fixed summation orders, no global scratch): up to 32
// tokens per-lane forms on the FP32 cores (one warp per rank; the product is
// a few loads per lane there), above that the tensor cores (tcgen05.mma with
// both operands from shared memory).  Each splits K over a thread-block
// cluster and adds the partial sums in rank order through distributed shared
// memory.
//
// Stream order: every form is launched WITHOUT programmatic stream
// serialisation, so they start only after every earlier kernel in the stream
// has completed, and each lets its dependent start at once.  The layer's
// launch that follows relies on this: it reads X and the weights without
// waiting and waits for this grid only before its first read of T.

#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc05.cuh"
#include "tmap.h"

namespace gptq {

namespace {

constexpr int kMaxSplits = 16;

// Up to 32 tokens: one warp per rank j, lane l taking 8-k chunk l of every
// 256-k piece of the CTA's k range (one 16-byte load of lora_a, one 16-byte
// load of X per token) into per-token FP32 sums, reduced across the warp by
// shuffles; the CTAs of a cluster split K and rank 0 adds their sums in rank
// order.  Two forms of the loop:
//  * up to 8 tokens (lanes form) X is read straight through L1 and the loop
//    has no barriers, so the loads of successive pieces overlap and a CTA
//    gets through its range in a few memory latencies even when only a few
//    CTAs run (launch_small);
//  * up to 32 tokens (staged form) each piece's X rows are staged in shared
//    memory once by all threads, two barriers per piece.
constexpr int SMALL_M = 32;
constexpr int LANES_M = 8;
constexpr int SMALL_WARPS = 8;  // ranks per CTA
constexpr int PIECE = 256;      // k per piece: one 8-k chunk per lane

// The common end of both forms: sums over the warp's lanes (fixed shuffle
// order), then over the cluster's CTAs in rank order in rank 0, then T.
template <int MB>
__device__ __forceinline__ void small_finish(float (&acc)[MB], float (*part)[MB], uint16_t* t,
                                             int M, int r, int split, int splits) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int m = 0; m < MB; ++m) {
    float v = acc[m];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
    if (lane == 0) part[warp][m] = v;
  }
  __syncthreads();
  // thread (w, m)
  const int w = threadIdx.x / MB, m = threadIdx.x % MB;
  const bool mine = threadIdx.x < SMALL_WARPS * MB;
  float sum = 0.0f;
  if (splits > 1) {
    cluster_sync_all();
    if (split == 0 && mine) {
      const uint32_t addr = smem_u32(&part[w][m]);
      for (int sp = 0; sp < splits; ++sp) sum += ld_dsmem_f32(map_to_rank(addr, (uint32_t)sp));
    }
    cluster_sync_all();  // no CTA leaves while rank 0 reads its shared memory
  } else if (mine) {
    sum = part[w][m];
  }
  const int jj = blockIdx.x * SMALL_WARPS + w;
  if (split == 0 && mine && m < M && jj < r)
    t[(int64_t)m * r + jj] = __half_as_ushort(__float2half_rn(sum));
}

// Lanes form, M <= LANES_M.
__global__ void __launch_bounds__(SMALL_WARPS * 32)
    lora_down_lanes_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ a,
                           uint16_t* __restrict__ t, int M, int K, int r, int splits) {
  __shared__ float part[SMALL_WARPS][LANES_M];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * SMALL_WARPS + warp;
  const int split = splits > 1 ? (int)cluster_ctarank() : 0;
  const int pieces = (K + PIECE - 1) / PIECE;
  // balanced: every split gets at least one piece (splits <= pieces)
  const int p_begin = split * pieces / splits, p_end = (split + 1) * pieces / splits;

  float acc[LANES_M];
#pragma unroll
  for (int m = 0; m < LANES_M; ++m) acc[m] = 0.0f;
  if (j < r) {
    const uint16_t* __restrict__ arow = a + (int64_t)j * K;
#pragma unroll 4
    for (int pc = p_begin; pc < p_end; ++pc) {
      const int k = pc * PIECE + 8 * lane;
      if (k < K) {  // K % 8 == 0: the chunk is whole
        const uint4 av = __ldg(reinterpret_cast<const uint4*>(arow + k));
        const float2 a0 = __half22float2(*reinterpret_cast<const __half2*>(&av.x));
        const float2 a1 = __half22float2(*reinterpret_cast<const __half2*>(&av.y));
        const float2 a2 = __half22float2(*reinterpret_cast<const __half2*>(&av.z));
        const float2 a3 = __half22float2(*reinterpret_cast<const __half2*>(&av.w));
#pragma unroll
        for (int m = 0; m < LANES_M; ++m)
          if (m < M)
            fma8(acc[m], __ldg(reinterpret_cast<const uint4*>(x + (int64_t)m * K + k)), a0, a1,
                 a2, a3);
      }
    }
  }
  small_finish<LANES_M>(acc, part, t, M, r, split, splits);
}

// Staged form, M <= SMALL_M.
__global__ void __launch_bounds__(SMALL_WARPS * 32)
    lora_down_staged_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ a,
                            uint16_t* __restrict__ t, int M, int K, int r, int splits) {
  constexpr int MB = SMALL_M;
  __shared__ __align__(16) uint16_t xs[MB][PIECE];
  __shared__ float part[SMALL_WARPS][MB];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * SMALL_WARPS + warp;
  const int split = splits > 1 ? (int)cluster_ctarank() : 0;
  const int pieces = (K + PIECE - 1) / PIECE;
  const int per = (pieces + splits - 1) / splits;
  const int p_begin = split * per, p_end = min(pieces, p_begin + per);

  float acc[MB];
#pragma unroll
  for (int m = 0; m < MB; ++m) acc[m] = 0.0f;
  for (int pc = p_begin; pc < p_end; ++pc) {
    const int k0 = pc * PIECE;
    // stage the piece's X rows (zero outside M and K)
    for (int i = threadIdx.x; i < MB * (PIECE / 8); i += SMALL_WARPS * 32) {
      const int m = i / (PIECE / 8), c = i % (PIECE / 8);
      uint4 v = make_uint4(0, 0, 0, 0);
      if (m < M && k0 + 8 * c < K)
        v = __ldg(reinterpret_cast<const uint4*>(x + (int64_t)m * K + k0 + 8 * c));
      *reinterpret_cast<uint4*>(&xs[m][8 * c]) = v;
    }
    __syncthreads();
    const int k = k0 + 8 * lane;
    if (j < r && k < K) {
      const uint4 av = __ldg(reinterpret_cast<const uint4*>(a + (int64_t)j * K + k));
      const float2 a0 = __half22float2(*reinterpret_cast<const __half2*>(&av.x));
      const float2 a1 = __half22float2(*reinterpret_cast<const __half2*>(&av.y));
      const float2 a2 = __half22float2(*reinterpret_cast<const __half2*>(&av.z));
      const float2 a3 = __half22float2(*reinterpret_cast<const __half2*>(&av.w));
#pragma unroll
      for (int m = 0; m < MB; ++m)
        if (m < M) fma8(acc[m], *reinterpret_cast<const uint4*>(&xs[m][8 * lane]), a0, a1, a2, a3);
    }
    __syncthreads();  // the piece is used before the next one is staged
  }
  small_finish<MB>(acc, part, t, M, r, split, splits);
}

// lanes: the lanes form (up to 8 tokens) on the free SMs when there are
// enough (the layer's launch after it then starts everywhere at once and its
// K stages overlap this one), else, like the staged form, split K over a
// cluster (at most 16) until the CTAs cover the SMs.
cudaError_t launch_small(bool lanes, const uint16_t* x, const uint16_t* lora_a, uint16_t* t,
                         int64_t M, int64_t K, int64_t r, int free_sms, cudaStream_t stream,
                         const DeviceInfo& dev) {
  const unsigned gr = (unsigned)((r + SMALL_WARPS - 1) / SMALL_WARPS);
  int splits = lanes && free_sms >= (int)gr ? free_sms / (int)gr : dev.num_sms / (int)gr;
  splits = std::max(1, std::min(kMaxSplits, splits));
  splits = std::min<int>(splits, (int)std::max<int64_t>(1, (K + PIECE - 1) / PIECE));
  const void* fn =
      lanes ? (const void*)lora_down_lanes_kernel : (const void*)lora_down_staged_kernel;
  if (splits > 8) {
    static std::once_flag once[2][64];
    static cudaError_t attr_err[2][64];
    const int d = dev.device & 63;
    std::call_once(once[lanes][d], [&] {
      attr_err[lanes][d] =
          cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    });
    if (attr_err[lanes][d] != cudaSuccess) splits = 8;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(gr, 1, (unsigned)splits);
  cfg.blockDim = dim3(SMALL_WARPS * 32, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = (unsigned)splits;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return lanes ? cudaLaunchKernelEx(&cfg, lora_down_lanes_kernel, x, lora_a, t, (int)M, (int)K,
                                    (int)r, splits)
               : cudaLaunchKernelEx(&cfg, lora_down_staged_kernel, x, lora_a, t, (int)M, (int)K,
                                    (int)r, splits);
}

// Above 32 tokens: the tensor cores.  T^T [r, M] = lora_a . X^T with both
// operands K-major FP16 tiles in shared memory (128-byte swizzle, by TMA):
// one CTA computes 128 ranks x 128 tokens into an FP32 accumulator in TMEM
// (tcgen05.mma, A and B from shared memory), 64 k per stage, four stages.
// When the tiles cannot fill the SMs, the CTAs of a cluster split K: each
// writes its tile to shared memory, and rank s adds rows s*128/S .. of every
// rank's tile in rank order (distributed shared memory) and stores them.
constexpr int TC_R = 128;    // ranks per CTA (MMA M; ranks past r read as zero)
constexpr int TC_T = 128;    // tokens per CTA (MMA N)
constexpr int TC_BK = 64;    // k per stage
constexpr int TC_STAGES = 4;
constexpr int TC_A_BYTES = TC_R * TC_BK * 2;
constexpr int TC_B_BYTES = TC_T * TC_BK * 2;
constexpr int TC_STAGE_BYTES = TC_A_BYTES + TC_B_BYTES;
constexpr int TC_THREADS = 192;  // warp 0: copies, warp 1: MMAs and TMEM, warps 2..5: read-out
constexpr int TC_RED_ROW = TC_T + 4;  // FP32 reduction rows, padded (16-byte stores, no conflicts)
constexpr int kTcMaxSplits = 8;
constexpr uint64_t kTcWaitNs = 4000000000ull;
constexpr uint64_t kTcDrainNs = 200000000ull;
static_assert(TC_R * TC_RED_ROW * 4 <= TC_STAGES * TC_STAGE_BYTES, "reduction tile fits the ring");

struct TcBars {
  uint64_t full[TC_STAGES];
  uint64_t empty[TC_STAGES];
  uint64_t dfull;
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(TC_THREADS, 1)
    lora_down_tc_kernel(const __grid_constant__ CUtensorMap a_map,
                        const __grid_constant__ CUtensorMap x_map, uint16_t* __restrict__ t,
                        int M, int K, int r, int splits, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  TcBars* bar = reinterpret_cast<TcBars*>(smem + TC_STAGES * TC_STAGE_BYTES);
  volatile int* abort_flag = &bar->abort_flag;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = splits > 1 ? (int)cluster_ctarank() : 0;
  const int t0 = blockIdx.x * TC_T, j0 = blockIdx.y * TC_R;
  const int KB = (K + TC_BK - 1) / TC_BK;
  // balanced split of the k stages: every CTA gets at least one (splits <=
  // KB), so every accumulator is written by its first MMA before it is read
  const int kb0 = (int)((int64_t)split * KB / splits);
  const int kb1 = (int)((int64_t)(split + 1) * KB / splits);
  const int n = kb1 - kb0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < TC_STAGES; ++s) {
      mbar_init(&bar->full[s], 1);
      mbar_init(&bar->empty[s], 1);
    }
    mbar_init(&bar->dfull, 1);
    bar->abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&a_map);
    prefetch_tensormap(&x_map);
  }
  __syncwarp();
  if (warp == 1) {
    tmem_alloc(&bar->tmem_base, TC_T);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      for (int i = 0; i < n; ++i) {
        if (!mbar_wait_bounded(&bar->empty[s], ph ^ 1u, abort_flag, kTcWaitNs)) {
          record_timeout(err, bar);
          break;
        }
        uint8_t* st = smem + s * TC_STAGE_BYTES;
        const int k0 = (kb0 + i) * TC_BK;
        mbar_arrive_expect_tx(&bar->full[s], TC_STAGE_BYTES);
        tma_load_2d(st, &a_map, k0, j0, &bar->full[s]);
        tma_load_2d(st + TC_A_BYTES, &x_map, k0, t0, &bar->full[s]);
        ++issued;
        if (++s == TC_STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (*abort_flag) {
        int never = 0;
        for (int j = issued - 1; j >= 0 && j >= issued - TC_STAGES; --j)
          mbar_wait_bounded(&bar->full[j % TC_STAGES], (uint32_t)(j / TC_STAGES) & 1u, &never,
                            kTcDrainNs);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    const uint32_t idesc = idesc_f16_f32(TC_R, TC_T);
    bool ok = true;
    int s = 0;
    uint32_t ph = 0;
    for (int i = 0; i < n && ok; ++i) {
      ok = __all_sync(0xffffffffu,
                      mbar_wait_bounded(&bar->full[s], ph, abort_flag, kTcWaitNs));
      if (!ok) break;
      tc_fence_after();
      const uint32_t st = smem_u32(smem + s * TC_STAGE_BYTES);
      const uint64_t a_desc = smem_desc_sw128(st), b_desc = smem_desc_sw128(st + TC_A_BYTES);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < TC_BK / 16; ++kk)
          mma_f16_ss(tmem, a_desc + (uint64_t)((kk * 32) >> 4), b_desc + (uint64_t)((kk * 32) >> 4),
                     idesc, (i | kk) != 0 ? 1u : 0u);
        mma_commit(&bar->empty[s]);
      }
      __syncwarp();
      if (++s == TC_STAGES) {
        s = 0;
        ph ^= 1u;
      }
    }
    if (!ok && lane == 0) {
      record_timeout(err, bar);
    }
    if (elect_one()) mma_commit(&bar->dfull);
    __syncwarp();
  }

  // read-out: warps 2..5, TMEM lane quarter warp % 4 (ranks j0 + 32q + lane)
  const bool reader = warp >= 2;
  const int q = warp & 3;
  const int j = j0 + 32 * q + lane;
  float* red = reinterpret_cast<float*>(smem);  // the ring is free once dfull completes
  bool ok = true;
  if (reader) {
    ok = __all_sync(0xffffffffu, mbar_wait_bounded<true>(&bar->dfull, 0, abort_flag, kTcWaitNs));
    if (!ok && lane == 0) {
      record_timeout(err, bar);
    }
  }
  if (reader && ok) {
    tc_fence_after();
#pragma unroll 1
    for (int c = 0; c < TC_T / 32; ++c) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + 32 * c, v);
      tmem_wait_ld();
      if (splits == 1) {
        if (j < r) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int tok = t0 + 32 * c + i;
            if (tok < M)
              t[(int64_t)tok * r + j] = __half_as_ushort(__float2half_rn(__uint_as_float(v[i])));
          }
        }
      } else {
        float* row = red + (32 * q + lane) * TC_RED_ROW + 32 * c;
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(row + i) =
              make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                          __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
      }
    }
  }
  if (splits > 1) {
    cluster_sync_all();  // every CTA's partial tile is in its shared memory
    if (reader) {
      // rank `split` adds rows split*RS .. of all ranks' tiles: thread i of
      // the 128 readers takes row split*RS + i / (128/RS), 128/(128/RS)
      // consecutive tokens of it
      const int RS = TC_R / splits;                 // rows per rank
      const int tpr = (TC_THREADS - 64) / RS;       // threads per row
      const int tid = threadIdx.x - 64;
      const int row = split * RS + tid / tpr;
      const int tw = TC_T / tpr;                    // tokens per thread
      const int tk0 = (tid % tpr) * tw;
      const int jr = j0 + row;
      for (int c = 0; c < tw; c += 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        const uint32_t addr = smem_u32(red + row * TC_RED_ROW + tk0 + c);
        for (int sp = 0; sp < splits; ++sp) {
          const uint32_t ra = map_to_rank(addr, (uint32_t)sp);
          acc.x += ld_dsmem_f32(ra);
          acc.y += ld_dsmem_f32(ra + 4);
          acc.z += ld_dsmem_f32(ra + 8);
          acc.w += ld_dsmem_f32(ra + 12);
        }
        const float vals[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int tok = t0 + tk0 + c + u;
          if (jr < r && tok < M)
            t[(int64_t)tok * r + jr] = __half_as_ushort(__float2half_rn(vals[u]));
        }
      }
    }
    cluster_sync_all();  // no CTA leaves while another reads its shared memory
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TC_T);
  }
}

cudaError_t launch_tc(const uint16_t* x, const uint16_t* lora_a, uint16_t* t, int64_t M,
                      int64_t K, int64_t r, cudaStream_t stream, const DeviceInfo& dev) {
  CUtensorMap a_map, x_map;
  if (!tensor_map_2d(&a_map, lora_a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)K, (uint64_t)r,
                     (uint64_t)K * 2, TC_BK, TC_R, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tensor_map_2d(&x_map, x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)K, (uint64_t)M,
                     (uint64_t)K * 2, TC_BK, TC_T, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const unsigned gm = (unsigned)((M + TC_T - 1) / TC_T), gr = (unsigned)((r + TC_R - 1) / TC_R);
  const int64_t tiles = (int64_t)gm * gr;
  const int64_t kb = (K + TC_BK - 1) / TC_BK;
  // a power-of-two K split (the reduction shares the 128 rows evenly) while
  // the tiles cannot fill the SMs
  int splits = 1;
  while (splits * 2 <= kTcMaxSplits && tiles * splits * 2 <= dev.num_sms && splits * 2 <= kb)
    splits *= 2;
  constexpr size_t smem = 1024 + (size_t)TC_STAGES * TC_STAGE_BYTES + 256;
  static std::once_flag once[64];
  static cudaError_t attr_err[64];
  const int d = dev.device & 63;
  std::call_once(once[d], [&] {
    attr_err[d] = cudaFuncSetAttribute(lora_down_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  });
  if (attr_err[d] != cudaSuccess) return attr_err[d];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(gm, gr, (unsigned)splits);
  cfg.blockDim = dim3(TC_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = (unsigned)splits;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, lora_down_tc_kernel, a_map, x_map, t, (int)M, (int)K, (int)r,
                            splits, dev.error_word);
}

}  // namespace

cudaError_t launch_lora_down(const uint16_t* x, const uint16_t* lora_a, uint16_t* t, int64_t M,
                             int64_t K, int64_t r, int free_sms, cudaStream_t stream,
                             const DeviceInfo& dev) {
  // up to 32 tokens the per-lane forms on the FP32 cores (an FP32 form with
  // shared-memory tiles took 14 us at M = 1, rank 32, stalled on barriers);
  // above, the tensor cores
  if (M <= LANES_M) return launch_small(true, x, lora_a, t, M, K, r, free_sms, stream, dev);
  if (M <= SMALL_M) return launch_small(false, x, lora_a, t, M, K, r, free_sms, stream, dev);
  return launch_tc(x, lora_a, t, M, K, r, stream, dev);
}

}  // namespace gptq
