// Decode kernel: Y[M, N] = X[M, K] . dequant(qweight, scales) for M <= 16.
//
// Operation: GPTQ-Pro README, "Runtime contract" and "Ampere kernel
// architecture" (fused small-M decode that reads the native int32 qweight,
// keeps scales resident, and reduces split-K partial sums deterministically).
// The Ampere design (four-warp output tiles, M <= 4) is prior art only; this
// kernel is laid out for sm_100a.
//
// * A CTA owns 64 output columns and a range of K.  One producer thread
//   streams, per stage (64 packed rows = 512 k), two TMA boxes of qweight
//   (32 columns x 64 rows each, stored with the 128-byte swizzle), one box of
//   the scale rows the stage needs and the X rows (bulk copies, 1088-byte
//   pitch) into a ring in shared memory, so tens of KB per SM stay in flight
//   without holding registers.
// * Eight consumer warps share every stage: warp w takes row quads 2w and
//   2w+1 (a row quad is four packed rows = 32 k).  A lane (q = lane/4,
//   c = lane%4) reads, for packed row 4j+c, the 16-byte vector at column chunk
//   chunk_of(q) of both boxes (eight columns; the chunk permutation makes the
//   eight lanes of each quarter-warp hit distinct banks through the swizzle)
//   and feeds mma.m16n8k16 with the weights as A (16 columns x 16 k) and X as
//   B (16 k x 8 tokens).  Which k sits in which MMA slot does not change the
//   sum as long as X uses the same order, so the (k, k+4) pairs of the
//   magic-number unpack are used as they come and X is permuted to match with
//   byte permutes, once per row quad for all eight columns.
// * Each weight is dequantised exactly as defined, fp16((q - 8) * s): 1024 + q
//   by a LOP3 into the FP16 mantissa of 1024, minus 1032 (exact), times the
//   group scale (one rounding).  Keeping the definition's per-weight rounding
//   matters: on inputs with large activation outliers, skipping it (scaling
//   FP32 partial sums per group instead) moves Y by up to ~1e-2 relative.
// * Split-K: the eight warps of a CTA and the `splits` CTAs of a thread-block
//   cluster (consecutive K ranges of the same columns) are reduced in a fixed
//   order through shared memory and distributed shared memory: bitwise
//   reproducible, no global scratch.
// * Programmatic dependent launch: before waiting for the previous kernel in
//   the stream, the producer only prefetches its first weight boxes into L2 (a
//   prefetch cannot observe stale data); every copy into shared memory and
//   every store of Y happens after the wait.  Once it has issued its last
//   copy, the producer lets the next kernel in the stream begin its prologue.
// * Every mbarrier wait is bounded in time; on expiry the kernel records
//   GPTQ_ERR_TIMEOUT in the device error word and winds down.
//
// Bytes per call: K*N/2 (qweight) + n_groups*N*2 (scales) + M*K*2 + M*N*2.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc05.cuh"
#include "tmap.h"

namespace gptq {

namespace {

constexpr int WC = 64;                  // output columns per CTA
constexpr int S_PITCH = WC * 2;         // 128 B per scale row
constexpr int kRqPerWarp = 2;           // row quads per consumer warp per stage
constexpr int kMaxStages = 8;
constexpr int kMaxConsumerWarps = 12;

// Geometry for NW consumer warps: a stage has RB = 8 NW packed rows (two row
// quads per warp); each 32-column qweight box of a stage is 32 x RB int32,
// stored with the 128-byte swizzle; X rows are padded to a pitch of 4 mod 8
// 16-byte units.
template <int NW>
struct Geo {
  static constexpr int RB = 4 * kRqPerWarp * NW;
  static constexpr int QW_BOX = 32 * RB * 4;
  static constexpr int X_PITCH = RB * 16 + 64;
  static constexpr int THREADS = (NW + 1) * 32;
};
constexpr int kRedStride = WC + 4;
constexpr uint64_t kWaitLimitNs = 4000000000ull;

struct DecodeShape {
  int nw;            // consumer warps
  int rb;            // packed rows per stage
  int stage_bytes;   // qweight + scales + X of one stage (1024-aligned)
  int s_off, x_off;
  int scale_rows;    // scale rows per stage (the scale box height)
  int stages;        // ring depth
  int smem_bytes;    // whole dynamic allocation
};

__host__ __device__ inline int align128(int v) { return (v + 127) & ~127; }
__host__ __device__ inline int align1024(int v) { return (v + 1023) & ~1023; }

// Scale rows a stage of `kspan` k (starting at a multiple of kspan) can
// touch: kspan / group when the group divides the span (the stages are then
// aligned to groups); otherwise the span may straddle one more boundary at
// each end.
__host__ __device__ inline int scale_rows_per_stage(int group_shift, int kspan) {
  if (group_shift >= 20) return 1;  // group -1: a single group
  const int g = 1 << group_shift;
  return kspan % g == 0 ? kspan / g : kspan / g + 2;
}

// M <= 8: twelve consumer warps (768-k stages); M <= 16: eight (512-k
// stages, the token tiles need more registers).  Two CTAs per SM either way.
inline DecodeShape decode_shape(int M, int group_shift) {
  DecodeShape d;
  d.nw = M <= 8 ? 12 : 8;
  d.rb = 8 * d.nw;
  const int qw_box = 32 * d.rb * 4, x_pitch = d.rb * 16 + 64;
  d.scale_rows = scale_rows_per_stage(group_shift, d.rb * 8);
  d.s_off = 2 * qw_box;
  d.x_off = d.s_off + align128(d.scale_rows * S_PITCH);
  d.stage_bytes = align1024(d.x_off + M * x_pitch);
  int s = (104 * 1024) / d.stage_bytes;
  d.stages = s < 3 ? 3 : (s > kMaxStages ? kMaxStages : s);
  d.smem_bytes = 1024 + d.stages * d.stage_bytes + 256;
  return d;
}

struct DecodeBars {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  int abort_flag;
};

__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* map, int32_t c0, int32_t c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1)
               : "memory");
}

// Shared-memory reads as ordinary C++ loads: ordered after the barrier waits
// (which clobber memory) but free to be scheduled among themselves.
__device__ __forceinline__ uint4 lds128(const uint8_t* p) {
  return *reinterpret_cast<const uint4*>(p);
}

__device__ __forceinline__ uint2 lds64(const uint8_t* p) {
  return *reinterpret_cast<const uint2*>(p);
}

__device__ __forceinline__ void record_timeout(int* err, volatile int* abort_flag) {
  atomicExch(err, kDeviceErrTimeout);
  *abort_flag = 1;
}

// Column chunk (of four columns) a lane reads: conflict-free against the
// 128-byte swizzle for the eight lanes of each quarter-warp.
__device__ __forceinline__ int chunk_of(int q) { return (q >> 1) + 4 * (q & 1); }

// TT: token tiles of 8 (1: M <= 8, 2: M <= 16).  PAIR_SCALE: the two row
// quads of a warp (64 consecutive k) lie in one group (every group size but
// 16 and 32), so one scale load serves both.  NW: consumer warps.
template <int TT, bool PAIR_SCALE, int NW>
__global__ void __launch_bounds__(Geo<NW>::THREADS) __maxnreg__(TT == 1 ? 72 : 96)
    decode_kernel(const __grid_constant__ CUtensorMap qw_map,
                  const __grid_constant__ CUtensorMap s_map, const uint16_t* __restrict__ x,
                  uint16_t* __restrict__ y, int M, int K, int N, int group_shift, int stages,
                  int stage_bytes, int s_off, int x_off, int scale_rows, int* err) {
  constexpr int RB = Geo<NW>::RB, QW_BOX = Geo<NW>::QW_BOX, X_PITCH = Geo<NW>::X_PITCH;
  constexpr int kConsumerWarps = NW, kThreads = Geo<NW>::THREADS;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array itself so that the
  // compiler keeps the shared address space (plain LDS, no generic loads)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  DecodeBars* bar = reinterpret_cast<DecodeBars*>(smem + stages * stage_bytes);
  volatile int* abort_flag = &bar->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_blk = blockIdx.x * WC;
  const int ncols = min(WC, N - n_blk);          // multiple of 8
  const int P = K >> 3;
  const int NS = (P + RB - 1) / RB;              // stages over all of K
  const int splits = gridDim.y;
  const int st_begin = (int)((int64_t)blockIdx.y * NS / splits);
  const int st_end = (int)((int64_t)(blockIdx.y + 1) * NS / splits);
  const int n_st = st_end - st_begin;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&bar->full[s], 1);
      mbar_init(&bar->empty[s], kConsumerWarps);  // every consumer warp reads every stage
    }
    bar->abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kConsumerWarps && lane == 0) {
    prefetch_tensormap(&qw_map);
    prefetch_tensormap(&s_map);
    // L2 prefetch of the first stages' weight boxes: safe before the wait
    const int pf = min(n_st, 3);
    for (int t = 0; t < pf; ++t) {
      tma_prefetch_l2_2d(&qw_map, n_blk, (st_begin + t) * RB);
      tma_prefetch_l2_2d(&qw_map, n_blk + 32, (st_begin + t) * RB);
    }
  }
  __syncthreads();
  grid_dependency_wait();

  // Consumer accumulators: acc[mt][tt] is m-tile mt, covering words 2mt (slot
  // q) and 2mt+1 (slot q+8) of the lane's eight columns (words 0-3 from box
  // 0, 4-7 from box 1).  The producer warp keeps its copy at zero.
  float acc[4][TT][4];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int tt = 0; tt < TT; ++tt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][tt][e] = 0.f;

  if (warp == kConsumerWarps) {
    // ---------------- producer (one lane) ----------------
    if (lane == 0) {
      int issued = 0;
      int s = 0;
      uint32_t ph = 0;
      for (int t = 0; t < n_st; ++t, s = (s + 1 == stages) ? 0 : s + 1, ph ^= (s == 0)) {
        if (!mbar_wait_bounded(&bar->empty[s], ph ^ 1u, abort_flag, kWaitLimitNs)) {
          record_timeout(err, abort_flag);
          break;
        }
        uint8_t* st = smem + s * stage_bytes;
        const int r0 = (st_begin + t) * RB;
        const int nrows = min(RB, P - r0);
        const int g0 = (int)(((int64_t)r0 * 8) >> group_shift);
        const uint32_t bytes = (uint32_t)(2 * QW_BOX + scale_rows * S_PITCH + M * nrows * 16);
        mbar_arrive_expect_tx(&bar->full[s], bytes);
        tma_load_2d(st, &qw_map, n_blk, r0, &bar->full[s]);
        tma_load_2d(st + QW_BOX, &qw_map, n_blk + 32, r0, &bar->full[s]);
        tma_load_2d(st + s_off, &s_map, n_blk, g0, &bar->full[s]);
        for (int m = 0; m < M; ++m)
          bulk_g2s(st + x_off + m * X_PITCH, x + (int64_t)m * K + (int64_t)r0 * 8,
                   (uint32_t)nrows * 16, &bar->full[s]);
        ++issued;
      }
      if (*abort_flag) {
        // wind down: wait (bounded) for the copies still landing in the ring
        int never = 0;
        for (int t = issued - 1; t >= 0 && t >= issued - stages; --t)
          mbar_wait_bounded(&bar->full[t % stages], (uint32_t)(t / stages) & 1u, &never,
                            200000000ull);
      }
      // all of this CTA's copies are issued: the next kernel in the stream may
      // start its prologue (it waits for this grid before touching its inputs)
      allow_dependent_launch();
    }
    __syncwarp();  // the whole warp reaches the CTA barrier below together
  } else {
    // ---------------- consumers ----------------
    const int q = lane >> 2, c = lane & 3;
    const int chunk = chunk_of(q);
    // byte offsets, inside a 128-byte swizzled row, of this lane's chunk in
    // rows with (row & 7) = c (even row quads) and c + 4 (odd row quads)
    const uint32_t off_even = (uint32_t)((chunk ^ c) << 4);
    const uint32_t off_odd = (uint32_t)((chunk ^ (c + 4)) << 4);
    bool x_ok[TT];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) x_ok[tt] = q + 8 * tt < M;


    bool ok = true;
    int s = 0;
    uint32_t ph = 0;
    for (int t = 0; t < n_st; ++t, s = (s + 1 == stages) ? 0 : s + 1, ph ^= (s == 0)) {
      ok = mbar_wait_bounded(&bar->full[s], ph, abort_flag, kWaitLimitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) record_timeout(err, abort_flag);
        break;
      }
      const uint8_t* st = smem + s * stage_bytes;
      const int r0 = (st_begin + t) * RB;
      const int nrows = min(RB, P - r0);
      const int g0 = (int)(((int64_t)r0 * 8) >> group_shift);
      const uint8_t* qw_lane = st + c * 128;  // row 4j + c: + 512 j
      const uint8_t* s_lane = st + s_off + chunk * 8;
      const uint8_t* x_lane[TT];
#pragma unroll
      for (int tt = 0; tt < TT; ++tt) x_lane[tt] = st + x_off + (q + 8 * tt) * X_PITCH + c * 16;
      uint32_t s2[8];

      // One row quad: 32 k x this lane's eight columns, eight tokens per tile.
      auto row_quad = [&](int j, bool full, bool load_scale) {
        const int row = 4 * j + c;
        const bool row_ok = full || row < nrows;
        if (load_scale) {
          // scale row of this lane's packed row within the stage's box; rows
          // past the end read a valid scale row and meet x = 0
          const int gl =
              row_ok ? (int)((((int64_t)(r0 + row)) * 8) >> group_shift) - g0 : 0;
          const uint2 sa = lds64(s_lane + gl * S_PITCH);        // columns of box 0
          const uint2 sb = lds64(s_lane + gl * S_PITCH + 64);   // columns of box 1
          s2[0] = prmt(sa.x, sa.x, 0x1010);
          s2[1] = prmt(sa.x, sa.x, 0x3232);
          s2[2] = prmt(sa.y, sa.y, 0x1010);
          s2[3] = prmt(sa.y, sa.y, 0x3232);
          s2[4] = prmt(sb.x, sb.x, 0x1010);
          s2[5] = prmt(sb.x, sb.x, 0x3232);
          s2[6] = prmt(sb.y, sb.y, 0x1010);
          s2[7] = prmt(sb.y, sb.y, 0x3232);
        }
        const uint8_t* qa = qw_lane + 512 * j + ((j & 1) ? off_odd : off_even);
        const uint4 w0 = lds128(qa);
        const uint4 w1 = lds128(qa + QW_BOX);
        uint32_t bx[TT][4];
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) {
          const uint4 xv = (row_ok && x_ok[tt]) ? lds128(x_lane[tt] + 64 * j)
                                                : make_uint4(0, 0, 0, 0);
          bx[tt][0] = prmt(xv.x, xv.z, 0x5410);  // (x0, x4)
          bx[tt][1] = prmt(xv.x, xv.z, 0x7632);  // (x1, x5)
          bx[tt][2] = prmt(xv.y, xv.w, 0x5410);  // (x2, x6)
          bx[tt][3] = prmt(xv.y, xv.w, 0x7632);  // (x3, x7)
        }
        const uint32_t wd[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            // column slots q (word 2mt) and q + 8 (word 2mt+1); MMA kk takes
            // the codes of bytes 0/2 (kk = 0) or 1/3 (kk = 1) of each word
            const uint32_t wa = kk ? (wd[2 * mt] >> 8) : wd[2 * mt];
            const uint32_t wb = kk ? (wd[2 * mt + 1] >> 8) : wd[2 * mt + 1];
            uint32_t a[4];
            a[0] = hmul2_rn(hsub2_rn(lop3_and_or(wa, 0x000F000Fu, kMagic1024), kMinus1032),
                            s2[2 * mt]);
            a[1] = hmul2_rn(hsub2_rn(lop3_and_or(wb, 0x000F000Fu, kMagic1024), kMinus1032),
                            s2[2 * mt + 1]);
            a[2] = hmul2_rn(
                hfma2_rn(lop3_and_or(wa, 0x00F000F0u, kMagic1024), kOneSixteenth, kMinus72),
                s2[2 * mt]);
            a[3] = hmul2_rn(
                hfma2_rn(lop3_and_or(wb, 0x00F000F0u, kMagic1024), kOneSixteenth, kMinus72),
                s2[2 * mt + 1]);
#pragma unroll
            for (int tt = 0; tt < TT; ++tt)
              mma_m16n8k16(acc[mt][tt], a, bx[tt][2 * kk], bx[tt][2 * kk + 1]);
          }
        }
      };

      const int j0 = kRqPerWarp * warp;
      if (nrows == RB) {
#pragma unroll
        for (int i = 0; i < kRqPerWarp; ++i) row_quad(j0 + i, true, !PAIR_SCALE || i == 0);
      } else {
#pragma unroll 1
        for (int i = 0; i < kRqPerWarp; ++i)
          if (4 * (j0 + i) < nrows) row_quad(j0 + i, false, true);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->empty[s]);
    }

    __syncwarp();
  }

  // Every stage has been consumed (so no copy is in flight): stash each
  // consumer warp's partial tile in the ring, then reduce in a fixed order.
  // Each CTA-wide barrier has a single call site reached by every thread.
  __syncthreads();
  constexpr int TOK = 8 * TT;
  if (warp < kConsumerWarps) {
    const int q = lane >> 2, c = lane & 3;
    float* red = reinterpret_cast<float*>(smem);  // [warp][tok][64 + 4]
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int tt = 0; tt < TT; ++tt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int wi = 2 * mt + (e >> 1);  // word index 0..7
          const int nl = 32 * (wi >> 2) + 4 * chunk_of(q) + (wi & 3);
          const int tok = 8 * tt + 2 * c + (e & 1);
          red[(warp * TOK + tok) * kRedStride + nl] = acc[mt][tt][e];
        }
  }
  __syncthreads();

  // fixed-order reduction: warps, then the cluster's CTAs
  static_assert(kConsumerWarps <= kMaxConsumerWarps, "reduction buffer");
  const float* red = reinterpret_cast<const float*>(smem);
  float* part = reinterpret_cast<float*>(smem) + kConsumerWarps * TOK * kRedStride;
  for (int idx = threadIdx.x; idx < TOK * WC; idx += kThreads) {
    const int tok = idx / WC, nl = idx - tok * WC;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) s += red[(w * TOK + tok) * kRedStride + nl];
    if (splits == 1) {
      if (tok < M && nl < ncols)
        y[(int64_t)tok * N + n_blk + nl] = __half_as_ushort(__float2half_rn(s));
    } else {
      part[idx] = s;
    }
  }
  if (splits > 1) {
    cluster_sync_all();
    const int rank = (int)cluster_ctarank();
    const int E = TOK * WC;
    const int begin = rank * E / splits, end = (rank + 1) * E / splits;
    const uint32_t base = smem_u32(part);
    for (int idx = begin + (int)threadIdx.x; idx < end; idx += kThreads) {
      const int tok = idx / WC, nl = idx - tok * WC;
      if (tok >= M || nl >= ncols) continue;
      float s = 0.f;
      for (int r = 0; r < splits; ++r) s += ld_dsmem_f32(map_to_rank(base + 4u * idx, r));
      y[(int64_t)tok * N + n_blk + nl] = __half_as_ushort(__float2half_rn(s));
    }
    cluster_sync_all();
  }
}

template <int TT, bool PAIR_SCALE, int NW>
cudaError_t launch_t(const CUtensorMap& qw_map, const CUtensorMap& s_map, const uint16_t* x,
                     uint16_t* y, int M, int K, int N, int group_shift, int splits,
                     const DecodeShape& d, cudaStream_t stream, const DeviceInfo& dev) {
  static std::once_flag once[64];
  static cudaError_t attr_err[64];
  const int di = dev.device & 63;
  std::call_once(once[di], [&] {
    attr_err[di] = cudaFuncSetAttribute(decode_kernel<TT, PAIR_SCALE, NW>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  });
  if (attr_err[di] != cudaSuccess) return attr_err[di];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((N + WC - 1) / WC), (unsigned)splits, 1);
  cfg.blockDim = dim3(Geo<NW>::THREADS, 1, 1);
  cfg.dynamicSmemBytes = (size_t)d.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (splits > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = 1;
    attr[n].val.clusterDim.y = (unsigned)splits;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, decode_kernel<TT, PAIR_SCALE, NW>, qw_map, s_map, x, y, M, K, N,
                            group_shift, d.stages, d.stage_bytes, d.s_off, d.x_off, d.scale_rows,
                            dev.error_word);
}

}  // namespace

int decode_pick_splits(int64_t M, int64_t K, int64_t N, const DeviceInfo& dev) {
  // The kernel is bound by the dequantisation work of the busiest SM, so
  // pick the split that minimises (CTAs on the busiest SM) x (stages per CTA)
  // plus one stage for the cluster reduction, among splits whose CTAs are all
  // resident at once (two per SM).  Ties go to the smaller split.
  const int64_t rb = 8 * (M <= 8 ? 12 : 8);
  const int64_t nblk = (N + WC - 1) / WC;
  const int64_t ns = ((K >> 3) + rb - 1) / rb;
  const int64_t sms = dev.num_sms;
  int best = 1;
  int64_t best_cost = -1;
  for (int s = 1; s <= 8; ++s) {
    if (s > 1 && (nblk * s > 2 * sms || ns < s)) break;
    const int64_t per_sm = (nblk * s + sms - 1) / sms;
    const int64_t cost = per_sm * ((ns + s - 1) / s) + (s > 1 ? 1 : 0);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

cudaError_t launch_decode(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                          uint16_t* y, int64_t M, int64_t K, int64_t N, int group_shift,
                          int splits, cudaStream_t stream, const DeviceInfo& dev) {
  if (splits <= 0) splits = decode_pick_splits(M, K, N, dev);
  const DecodeShape d = decode_shape((int)M, group_shift);
  // the reduction reuses the ring: it must fit
  const int red_bytes = (kMaxConsumerWarps * 16 * kRedStride + 16 * WC) * 4;
  if (d.stages * d.stage_bytes < red_bytes) return cudaErrorInvalidValue;
  const int iM = (int)M, iK = (int)K, iN = (int)N;
  const int64_t n_groups = (group_shift == 62 || (int64_t(1) << group_shift) >= K)
                               ? 1 : (K + (int64_t(1) << group_shift) - 1) >> group_shift;
  CUtensorMap qw_map, s_map;
  if (!tensor_map_2d(&qw_map, qweight, CU_TENSOR_MAP_DATA_TYPE_INT32, (uint64_t)N,
                     (uint64_t)(K / 8), (uint64_t)N * 4, 32, (uint32_t)d.rb,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tensor_map_2d(&s_map, scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, (uint64_t)N,
                     (uint64_t)n_groups, (uint64_t)N * 2, WC, (uint32_t)d.scale_rows,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  // a warp's two row quads (64 k) share one group for every group size >= 64
  const bool pair_scale = group_shift >= 6;
#define GPTQ_DECODE_LAUNCH(TT_, PS_, NW_) \
  launch_t<TT_, PS_, NW_>(qw_map, s_map, x, y, iM, iK, iN, group_shift, splits, d, stream, dev)
  if (M <= 8)
    return pair_scale ? GPTQ_DECODE_LAUNCH(1, true, 12) : GPTQ_DECODE_LAUNCH(1, false, 12);
  return pair_scale ? GPTQ_DECODE_LAUNCH(2, true, 8) : GPTQ_DECODE_LAUNCH(2, false, 8);
#undef GPTQ_DECODE_LAUNCH
}

}  // namespace gptq
