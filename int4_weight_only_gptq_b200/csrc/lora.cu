// The LoRA adapter's down-projection: T[M, r] = fp16(X[M, K] . lora_a[r, K]^T).
//
// GPTQ-Pro README, "Runtime contract": adapters are LoRA on the linear path;
// the adapter's own output is FP16 (its dtype), summed here in FP32.  T then
// enters the prefill pair kernel as extra K of the layer's product
// (prefill_pair.cu), where T . lora_b^T is added to the FP32 accumulator.
//
// This product is at most rank/N of the layer's work (well under 1 % for the
// usual ranks), so it runs on the FP32 cores: one CTA computes 32 tokens x 32
// ranks, streaming 64-k chunks of X and lora_a through shared memory (as
// FP32, with three chunks in flight in registers: at small M this product is
// a few chunks per CTA, and memory latency, not arithmetic, sets its time).  When there are fewer tiles than twice the SMs, the CTAs of a
// thread-block cluster (up to 16) split K and the partial sums are added in a
// fixed order (rank 0, 1, ...) through distributed shared memory, so T is the
// same on every call.

#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace gptq {

namespace {

constexpr int MT = 32;           // tokens per CTA
constexpr int RT = 32;           // ranks per CTA (one per lane)
constexpr int KC = 64;           // k per shared-memory chunk
constexpr int THREADS = 256;     // warp w: tokens 4w .. 4w+3; lane: one rank
constexpr int TOK_PER_WARP = MT / (THREADS / 32);
constexpr int A_ROW = KC + 4;    // padded FP32 row: 16-byte loads by 8 lanes hit 32 banks
constexpr int WORDS = MT * KC / 2 / THREADS;  // 32-bit words of each chunk per thread
constexpr int kMaxSplits = 16;
constexpr int PF = 3;  // chunks in flight per thread
static_assert(RT * KC / 2 / THREADS == WORDS, "X and lora_a chunks have the same size");

// This thread's words of chunk c: X rows m0.., lora_a rows j0.. (zero outside
// M, r and K).
__device__ __forceinline__ void load_chunk(const uint16_t* __restrict__ x,
                                           const uint16_t* __restrict__ a, int M, int K, int r,
                                           int m0, int j0, int c, uint32_t (&xv)[WORDS],
                                           uint32_t (&av)[WORDS]) {
  const int k0 = c * KC;
#pragma unroll
  for (int u = 0; u < WORDS; ++u) {
    const int i = threadIdx.x + u * THREADS;
    const int row = i / (KC / 2), k = k0 + 2 * (i % (KC / 2));
    const int m = m0 + row, j = j0 + row;
    xv[u] = (m < M && k < K) ? __ldg(reinterpret_cast<const unsigned int*>(x + (int64_t)m * K + k))
                             : 0u;
    av[u] = (j < r && k < K) ? __ldg(reinterpret_cast<const unsigned int*>(a + (int64_t)j * K + k))
                             : 0u;
  }
}

__global__ void __launch_bounds__(THREADS)
    lora_down_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ a,
                     uint16_t* __restrict__ t, int M, int K, int r, int splits) {
  __shared__ __align__(16) float xs[MT][KC];     // X chunk in FP32
  __shared__ __align__(16) float as[RT][A_ROW];  // lora_a chunk in FP32 (padded rows)
  __shared__ float part[THREADS][TOK_PER_WARP];

  // The layer launch that reads T may start now: it waits for this grid's
  // completion before its first read of T, and every CTA of this grid is
  // resident once all have passed this point, so the early start cannot keep
  // any of them from an SM.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * MT, j0 = blockIdx.y * RT;
  const int split = splits > 1 ? (int)cluster_ctarank() : 0;  // the cluster spans z
  // this CTA's k range, whole chunks
  const int chunks = (K + KC - 1) / KC;
  const int per = (chunks + splits - 1) / splits;
  const int c_begin = split * per, c_end = min(chunks, c_begin + per);

  float acc[TOK_PER_WARP] = {};
  // PF chunks in flight in registers: ring slot u holds chunk c_begin + u
  // (mod PF); a slot is refilled as soon as its chunk is in shared memory
  uint32_t xv[PF][WORDS], av[PF][WORDS];
#pragma unroll
  for (int u = 0; u < PF; ++u)
    if (c_begin + u < c_end) load_chunk(x, a, M, K, r, m0, j0, c_begin + u, xv[u], av[u]);
  for (int c0 = c_begin; c0 < c_end; c0 += PF) {
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      const int c = c0 + u;
      if (c >= c_end) break;
      // store chunk c (FP32), refill its slot with chunk c + PF, compute
#pragma unroll
      for (int w = 0; w < WORDS; ++w) {
        const int i = threadIdx.x + w * THREADS;
        const int row = i / (KC / 2), col2 = i % (KC / 2);
        *reinterpret_cast<float2*>(&xs[row][2 * col2]) =
            __half22float2(*reinterpret_cast<const __half2*>(&xv[u][w]));
        *reinterpret_cast<float2*>(&as[row][2 * col2]) =
            __half22float2(*reinterpret_cast<const __half2*>(&av[u][w]));
      }
      __syncthreads();
      if (c + PF < c_end) load_chunk(x, a, M, K, r, m0, j0, c + PF, xv[u], av[u]);
#pragma unroll 4
      for (int k = 0; k < KC; k += 4) {
        const float4 a4 = *reinterpret_cast<const float4*>(&as[lane][k]);
#pragma unroll
        for (int q = 0; q < TOK_PER_WARP; ++q) {
          const float4 x4 = *reinterpret_cast<const float4*>(&xs[TOK_PER_WARP * warp + q][k]);
          acc[q] = fmaf(x4.x, a4.x, acc[q]);
          acc[q] = fmaf(x4.y, a4.y, acc[q]);
          acc[q] = fmaf(x4.z, a4.z, acc[q]);
          acc[q] = fmaf(x4.w, a4.w, acc[q]);
        }
      }
      __syncthreads();
    }
  }

  // partial sums of this CTA, then (split-K) the fixed-order sum over the
  // cluster's CTAs in rank 0
#pragma unroll
  for (int q = 0; q < TOK_PER_WARP; ++q) part[threadIdx.x][q] = acc[q];
  if (splits > 1) {
    cluster_sync_all();  // every CTA's partial sums are in its shared memory
    if (split == 0) {
      const uint32_t mine = smem_u32(&part[threadIdx.x][0]);
#pragma unroll
      for (int q = 0; q < TOK_PER_WARP; ++q) acc[q] = 0.0f;
      for (int s = 0; s < splits; ++s) {
        const uint32_t addr = map_to_rank(mine, (uint32_t)s);
#pragma unroll
        for (int q = 0; q < TOK_PER_WARP; ++q) acc[q] += ld_dsmem_f32(addr + 4u * q);
      }
    }
    cluster_sync_all();  // no CTA leaves while rank 0 reads its shared memory
  }
  if (split == 0) {
    const int j = j0 + lane;
#pragma unroll
    for (int q = 0; q < TOK_PER_WARP; ++q) {
      const int m = m0 + TOK_PER_WARP * warp + q;
      if (m < M && j < r) t[(int64_t)m * r + j] = __half_as_ushort(__float2half_rn(acc[q]));
    }
  }
}

// Up to 32 tokens: one warp per rank j.  The CTA's k range goes in pieces
// of 256: the piece's X rows are staged in shared memory once (16-byte
// loads by all threads), then lane l of each warp takes k chunk l of the
// piece (eight values: one 16-byte load of lora_a, one 16-byte shared load
// per token) into per-token FP32 sums, reduced across the warp by shuffles;
// the CTAs of a cluster split K and rank 0 adds their sums in rank order.
// Two barriers per 256 k, against two per 64 k in the tiled form.
constexpr int SMALL_M = 32;
constexpr int SMALL_WARPS = 8;  // ranks per CTA
constexpr int PIECE = 256;      // k per staged piece: one 8-k chunk per lane

template <int MB>  // token bound: M <= MB
__global__ void __launch_bounds__(SMALL_WARPS * 32)
    lora_down_small_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ a,
                           uint16_t* __restrict__ t, int M, int K, int r, int splits) {
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
      for (int m = 0; m < MB; ++m) {
        if (m < M) {
          const uint4 xv = *reinterpret_cast<const uint4*>(&xs[m][8 * lane]);
          const float2 x0 = __half22float2(*reinterpret_cast<const __half2*>(&xv.x));
          const float2 x1 = __half22float2(*reinterpret_cast<const __half2*>(&xv.y));
          const float2 x2 = __half22float2(*reinterpret_cast<const __half2*>(&xv.z));
          const float2 x3 = __half22float2(*reinterpret_cast<const __half2*>(&xv.w));
          float sm = acc[m];
          sm = fmaf(x0.x, a0.x, sm);
          sm = fmaf(x0.y, a0.y, sm);
          sm = fmaf(x1.x, a1.x, sm);
          sm = fmaf(x1.y, a1.y, sm);
          sm = fmaf(x2.x, a2.x, sm);
          sm = fmaf(x2.y, a2.y, sm);
          sm = fmaf(x3.x, a3.x, sm);
          sm = fmaf(x3.y, a3.y, sm);
          acc[m] = sm;
        }
      }
    }
    __syncthreads();  // the piece is used before the next one is staged
  }
  // sums over the warp's lanes (fixed shuffle order), lane 0 keeps them
#pragma unroll
  for (int m = 0; m < MB; ++m) {
    float v = acc[m];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
    if (lane == 0) part[warp][m] = v;
  }
  __syncthreads();
  // then over the cluster's CTAs in rank order, in rank 0; thread (w, m)
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

template <int MB>
cudaError_t launch_small(const uint16_t* x, const uint16_t* lora_a, uint16_t* t, int64_t M,
                         int64_t K, int64_t r, cudaStream_t stream, const DeviceInfo& dev) {
  const unsigned gr = (unsigned)((r + SMALL_WARPS - 1) / SMALL_WARPS);
  // split K over a cluster until the CTAs cover the SMs (at most 16)
  int splits = (int)std::min<int64_t>(kMaxSplits, std::max<int64_t>(1, dev.num_sms / gr));
  splits = std::min<int>(splits, (int)std::max<int64_t>(1, (K + PIECE - 1) / PIECE));
  if (splits > 8) {
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    const int d = dev.device & 63;
    std::call_once(once[d], [&] {
      attr_err[d] = cudaFuncSetAttribute(lora_down_small_kernel<MB>,
                                         cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    });
    if (attr_err[d] != cudaSuccess) splits = 8;
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
  return cudaLaunchKernelEx(&cfg, lora_down_small_kernel<MB>, x, lora_a, t, (int)M, (int)K,
                            (int)r, splits);
}

}  // namespace

cudaError_t launch_lora_down(const uint16_t* x, const uint16_t* lora_a, uint16_t* t, int64_t M,
                             int64_t K, int64_t r, cudaStream_t stream, const DeviceInfo& dev) {
  // up to 32 tokens the per-lane form (measured at M = 1, rank 32: 5.5 us
  // against 14 us for the tiled form, which stalls on barriers there)
  if (M <= 8) return launch_small<8>(x, lora_a, t, M, K, r, stream, dev);
  if (M <= SMALL_M) return launch_small<SMALL_M>(x, lora_a, t, M, K, r, stream, dev);
  const unsigned gm = (unsigned)((M + MT - 1) / MT), gr = (unsigned)((r + RT - 1) / RT);
  const int64_t tiles = (int64_t)gm * gr;
  const int chunks = (int)((K + KC - 1) / KC);
  // split K over a cluster when the tiles alone cannot fill the SMs twice
  int splits = (int)std::min<int64_t>(kMaxSplits, std::max<int64_t>(1, 2 * dev.num_sms / tiles));
  splits = std::min(splits, chunks);
  if (splits > 8) {
    // clusters above the portable size of 8 have to be allowed per kernel
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    const int d = dev.device & 63;
    std::call_once(once[d], [&] {
      attr_err[d] = cudaFuncSetAttribute(lora_down_kernel,
                                         cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    });
    if (attr_err[d] != cudaSuccess) splits = 8;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(gm, gr, (unsigned)splits);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = (unsigned)splits;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, lora_down_kernel, x, lora_a, t, (int)M, (int)K, (int)r, splits);
}

}  // namespace gptq
