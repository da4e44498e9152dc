// The LoRA adapter's down-projection: T[M, r] = fp16(X[M, K] . lora_a[r, K]^T).
//
// GPTQ-Pro README, "Runtime contract": adapters are LoRA on the linear path;
// the adapter's own output is FP16 (its dtype), summed here in FP32.  T then
// enters the prefill pair kernel as extra K of the layer's product
// (prefill_pair.cu), where T . lora_b^T is added to the FP32 accumulator.
//
// This product is at most rank/N of the layer's work (well under 1 % for the
// usual ranks), so it runs on the FP32 cores: one CTA computes 32 tokens x 32
// ranks, streaming 64-k chunks of X and lora_a through shared memory.  When
// there are fewer tiles than SMs, the CTAs of a thread-block cluster split K
// and the partial sums are added in a fixed order (rank 0, 1, ...) through
// distributed shared memory, so T is the same on every call.

#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace gptq {

namespace {

constexpr int MT = 32;           // tokens per CTA
constexpr int RT = 32;           // ranks per CTA (one per lane)
constexpr int KC = 64;           // k per shared-memory chunk
constexpr int THREADS = 256;     // warp w: tokens 4w .. 4w+3; lane: one rank
constexpr int TOK_PER_WARP = MT / (THREADS / 32);
constexpr int A_ROW_WORDS = KC / 2 + 1;  // padded: lane j reads row j conflict-free
constexpr int kMaxSplits = 8;

__global__ void __launch_bounds__(THREADS)
    lora_down_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ a,
                     uint16_t* __restrict__ t, int M, int K, int r, int splits) {
  __shared__ uint32_t xs[MT][KC / 2];       // X chunk, half2 per word
  __shared__ uint32_t as[RT][A_ROW_WORDS];  // lora_a chunk, half2 per word (padded rows)
  __shared__ float part[THREADS][TOK_PER_WARP];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * MT, j0 = blockIdx.y * RT;
  const int split = splits > 1 ? (int)cluster_ctarank() : 0;  // the cluster spans z
  // this CTA's k range, whole chunks
  const int chunks = (K + KC - 1) / KC;
  const int per = (chunks + splits - 1) / splits;
  const int c_begin = split * per, c_end = min(chunks, c_begin + per);

  float acc[TOK_PER_WARP] = {};
  for (int c = c_begin; c < c_end; ++c) {
    const int k0 = c * KC;
    // X chunk: 32 rows x 64 k, 32-bit words (zero outside M and K)
    for (int i = threadIdx.x; i < MT * KC / 2; i += THREADS) {
      const int row = i / (KC / 2), w = i % (KC / 2);
      const int m = m0 + row, k = k0 + 2 * w;
      uint32_t v = 0;
      if (m < M && k < K) v = *reinterpret_cast<const uint32_t*>(x + (int64_t)m * K + k);
      xs[row][w] = v;
    }
    // lora_a chunk: 32 ranks x 64 k (zero outside r and K)
    for (int i = threadIdx.x; i < RT * KC / 2; i += THREADS) {
      const int row = i / (KC / 2), w = i % (KC / 2);
      const int j = j0 + row, k = k0 + 2 * w;
      uint32_t v = 0;
      if (j < r && k < K) v = *reinterpret_cast<const uint32_t*>(a + (int64_t)j * K + k);
      as[row][w] = v;
    }
    __syncthreads();
#pragma unroll 8
    for (int w = 0; w < KC / 2; ++w) {
      const float2 av = __half22float2(*reinterpret_cast<const __half2*>(&as[lane][w]));
#pragma unroll
      for (int q = 0; q < TOK_PER_WARP; ++q) {
        const float2 xv =
            __half22float2(*reinterpret_cast<const __half2*>(&xs[TOK_PER_WARP * warp + q][w]));
        acc[q] = fmaf(xv.x, av.x, acc[q]);
        acc[q] = fmaf(xv.y, av.y, acc[q]);
      }
    }
    __syncthreads();
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

}  // namespace

cudaError_t launch_lora_down(const uint16_t* x, const uint16_t* lora_a, uint16_t* t, int64_t M,
                             int64_t K, int64_t r, cudaStream_t stream, const DeviceInfo& dev) {
  const unsigned gm = (unsigned)((M + MT - 1) / MT), gr = (unsigned)((r + RT - 1) / RT);
  const int64_t tiles = (int64_t)gm * gr;
  const int chunks = (int)((K + KC - 1) / KC);
  // split K over a cluster when the tiles alone cannot fill the SMs
  int splits = (int)std::min<int64_t>(kMaxSplits, std::max<int64_t>(1, dev.num_sms / tiles));
  splits = std::min(splits, chunks);
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
