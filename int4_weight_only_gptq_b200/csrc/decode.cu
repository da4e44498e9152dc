// Decode kernel: Y[M, N] = X[M, K] . dequant(qweight, scales) for M <= 16.
//
// Operation: GPTQ-Pro README, "Runtime contract" and "Ampere kernel
// architecture" (fused small-M decode that reads the native int32 qweight,
// keeps scales close, and reduces split-K partial sums deterministically).
// The Ampere design (four-warp output tiles, M <= 4) is prior art only; this
// kernel is laid out for sm_100a:
//
// * Work unit: a "row quad" (four packed rows = 32 k) by 32 or 64 columns per
//   warp.  Lane (q = lane/4, c = lane%4) loads the 16-byte qweight vector of
//   packed row 4r+c, columns n + 4q .. n + 4q + 3: for each c the eight lanes
//   read 128 contiguous bytes, so every warp load is four full 128-byte lines.
// * The eight codes of a word are unpacked in registers straight into the
//   A fragment of mma.m16n8k16 (weights as A: 16 columns x 16 k; X as B:
//   16 k x 8 tokens).  The k order inside one MMA does not change the sum as
//   long as X uses the same order, so the natural (k, k+4) pairs of the
//   magic-number unpack are used as they come and X is permuted to match with
//   two byte-permutes per register.  Weights are the exact FP16 dequantised
//   values (one rounding), accumulation is FP32 on the tensor cores, which
//   keeps the CUDA-core work per weight to a handful of ALU operations.
// * Split-K: the eight warps of a CTA take consecutive K ranges of the same
//   columns; `splits` CTAs of a thread-block cluster take consecutive K ranges
//   of the same column block.  Partial sums are reduced in a fixed order
//   through shared memory and then distributed shared memory, so results are
//   bitwise reproducible and no global scratch is needed.
//
// Bytes per call: K*N/2 (qweight) + n_groups*N*2 (scales) + M*K*2 + M*N*2.
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace gptq {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

template <int TT, int WCV>
struct DecodeFrag {
  uint4 w[WCV];   // qweight words, columns col[v] .. col[v] + 3
  uint2 s[WCV];   // their scales (four halves)
  uint4 xv[TT];   // X[token q + 8 tt][8 i .. 8 i + 7]
};

// TT: token tiles of 8 (1: M <= 8, 2: M <= 16); WCV: 16-byte column vectors per
// lane (columns per CTA = 32 * WCV).
template <int TT, int WCV>
__global__ void __launch_bounds__(kThreads, 2)
    decode_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ qweight,
                  const uint16_t* __restrict__ scales, uint16_t* __restrict__ y, int M, int K,
                  int N, int group_shift) {
  constexpr int WC = 32 * WCV;
  constexpr int TOK = 8 * TT;
  constexpr int RED_STRIDE = WC + 4;
  __shared__ float red[kWarps][TOK][RED_STRIDE];
  __shared__ float part[TOK * WC];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = lane >> 2, c = lane & 3;
  const int n_blk = blockIdx.x * WC;
  const int splits = gridDim.y;
  const int P = K >> 3;                 // packed rows
  const int RQ = (P + 3) >> 2;          // row quads (the last may be half full)
  const int split = blockIdx.y * kWarps + warp;
  const int S = splits * kWarps;
  const int rq_begin = (int)((int64_t)split * RQ / S);
  const int rq_end = (int)((int64_t)(split + 1) * RQ / S);

  int col[WCV];
  bool col_ok[WCV];
#pragma unroll
  for (int v = 0; v < WCV; ++v) {
    col[v] = n_blk + 32 * v + 4 * q;
    col_ok[v] = col[v] < N;
  }

  float acc[WCV][2][TT][4];
#pragma unroll
  for (int v = 0; v < WCV; ++v)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int tt = 0; tt < TT; ++tt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[v][mt][tt][e] = 0.f;

  auto fetch = [&](int r, DecodeFrag<TT, WCV>& f) {
    const int i = 4 * r + c;
    const bool row_ok = i < P;
    const int64_t g = ((int64_t)i * 8) >> group_shift;
#pragma unroll
    for (int v = 0; v < WCV; ++v) {
      if (row_ok && col_ok[v]) {
        f.w[v] = ld_stream_v4(qweight + (int64_t)i * N + col[v]);
        f.s[v] = ld_nc_v2(scales + g * N + col[v]);
      } else {
        f.w[v] = make_uint4(0, 0, 0, 0);
        f.s[v] = make_uint2(0, 0);
      }
    }
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
      const int tok = q + 8 * tt;
      if (row_ok && tok < M)
        f.xv[tt] = ld_nc_v4(x + (int64_t)tok * K + (int64_t)i * 8);
      else
        f.xv[tt] = make_uint4(0, 0, 0, 0);
    }
  };

  auto compute = [&](const DecodeFrag<TT, WCV>& f) {
    uint32_t bx[TT][4];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
      bx[tt][0] = prmt(f.xv[tt].x, f.xv[tt].z, 0x5410);  // (x0, x4)
      bx[tt][1] = prmt(f.xv[tt].x, f.xv[tt].z, 0x7632);  // (x1, x5)
      bx[tt][2] = prmt(f.xv[tt].y, f.xv[tt].w, 0x5410);  // (x2, x6)
      bx[tt][3] = prmt(f.xv[tt].y, f.xv[tt].w, 0x7632);  // (x3, x7)
    }
#pragma unroll
    for (int v = 0; v < WCV; ++v) {
      const uint32_t words[4] = {f.w[v].x, f.w[v].y, f.w[v].z, f.w[v].w};
      const uint32_t s01 = f.s[v].x, s23 = f.s[v].y;
      const uint32_t s2[4] = {prmt(s01, s01, 0x1010), prmt(s01, s01, 0x3232),
                              prmt(s23, s23, 0x1010), prmt(s23, s23, 0x3232)};
      uint32_t p[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) dequant_word_paired(words[j], s2[j], p[j]);
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const int a = 2 * mt, b = 2 * mt + 1;  // column slots q and q + 8
#pragma unroll
        for (int st = 0; st < 2; ++st) {
          const uint32_t afrag[4] = {p[a][2 * st], p[b][2 * st], p[a][2 * st + 1],
                                     p[b][2 * st + 1]};
#pragma unroll
          for (int tt = 0; tt < TT; ++tt)
            mma_m16n8k16(acc[v][mt][tt], afrag, bx[tt][2 * st], bx[tt][2 * st + 1]);
        }
      }
    }
  };

  if (rq_begin < rq_end) {
    DecodeFrag<TT, WCV> cur, nxt;
    fetch(rq_begin, cur);
    for (int r = rq_begin; r < rq_end; ++r) {
      if (r + 1 < rq_end) fetch(r + 1, nxt);
      compute(cur);
      cur = nxt;
    }
  }

  // Accumulator (v, mt, tt, e) holds column slot q (+8 for e >= 2) and token
  // 2c + (e & 1) of its tile; slot q maps to column 4q + 2mt, slot q + 8 to
  // column 4q + 2mt + 1 within vector v.
#pragma unroll
  for (int v = 0; v < WCV; ++v)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int tt = 0; tt < TT; ++tt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int nl = 32 * v + 4 * q + 2 * mt + (e >> 1);
          const int tok = 8 * tt + 2 * c + (e & 1);
          red[warp][tok][nl] = acc[v][mt][tt][e];
        }
  __syncthreads();

  for (int idx = threadIdx.x; idx < TOK * WC; idx += kThreads) {
    const int tok = idx / WC, nl = idx - tok * WC;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += red[w][tok][nl];  // fixed order
    if (splits == 1) {
      if (tok < M && n_blk + nl < N) y[(int64_t)tok * N + n_blk + nl] = __half_as_ushort(__float2half_rn(s));
    } else {
      part[idx] = s;
    }
  }
  if (splits > 1) {
    cluster_sync_all();  // every CTA's partial is visible cluster-wide
    const int rank = (int)cluster_ctarank();
    const int E = TOK * WC;
    const int begin = rank * E / splits, end = (rank + 1) * E / splits;
    const uint32_t base = smem_u32(part);
    for (int idx = begin + threadIdx.x; idx < end; idx += kThreads) {
      const int tok = idx / WC, nl = idx - tok * WC;
      if (tok >= M || n_blk + nl >= N) continue;
      float s = 0.f;
      for (int r = 0; r < splits; ++r) s += ld_dsmem_f32(map_to_rank(base + 4u * idx, r));
      y[(int64_t)tok * N + n_blk + nl] = __half_as_ushort(__float2half_rn(s));
    }
    cluster_sync_all();  // keep every CTA's shared memory alive until read
  }
}

template <int TT, int WCV>
cudaError_t launch_decode_t(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                            uint16_t* y, int64_t M, int64_t K, int64_t N, int group_shift,
                            int splits, cudaStream_t stream) {
  constexpr int WC = 32 * WCV;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((N + WC - 1) / WC), (unsigned)splits, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = (unsigned)splits;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel<TT, WCV>, x, qweight, scales, y, (int)M, (int)K,
                            (int)N, group_shift);
}

}  // namespace

int decode_pick_splits(int64_t M, int64_t K, int64_t N, const DeviceInfo& dev) {
  // Fill the machine with CTAs of 8 warps; each warp should keep at least
  // three row quads (96 k) of work so the loads can be pipelined.
  (void)M;
  const int64_t WC = 64;
  const int64_t nblk = (N + WC - 1) / WC;
  const int64_t rq = ((K >> 3) + 3) >> 2;
  const int64_t slots = (int64_t)dev.num_sms * 2;
  int best = 1;
  double best_eff = -1.0;
  for (int s = 1; s <= 8; ++s) {
    if (s > 1 && rq < (int64_t)s * kWarps * 3) break;
    const int64_t ctas = nblk * s;
    const int64_t waves = (ctas + slots - 1) / slots;
    const double eff = (double)ctas / (double)(waves * slots);
    if (eff > best_eff + 0.02) {
      best_eff = eff;
      best = s;
    }
  }
  return best;
}

cudaError_t launch_decode(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                          uint16_t* y, int64_t M, int64_t K, int64_t N, int group_shift,
                          int splits, cudaStream_t stream, const DeviceInfo& dev) {
  if (splits <= 0) splits = decode_pick_splits(M, K, N, dev);
  if (M <= 8)
    return launch_decode_t<1, 2>(x, qweight, scales, y, M, K, N, group_shift, splits, stream);
  return launch_decode_t<2, 2>(x, qweight, scales, y, M, K, N, group_shift, splits, stream);
}

}  // namespace gptq
