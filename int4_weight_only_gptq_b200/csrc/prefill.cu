// Single-CTA prefill kernel: Y[M, N] = X[M, K] . dequant(qweight, scales) on
// the 5th-generation tensor cores (tcgen05) with TMEM accumulators, and the
// prefill dispatcher.
//
// Operation: GPTQ-Pro README, "Runtime contract" and "Ampere kernel
// architecture" (tensor-core prefill with FP32 accumulation that reads the
// native int32 qweight; predicated tails; FP16 output).  The Ampere design
// (cp.async staging, mma.sync) is prior art only.
//
// Above 32 tokens the dispatcher below sends every call to the persistent
// CTA-pair kernel (prefill_pair.cu).  This kernel takes the prefill path at
// M <= 32, which only a caller that forces the prefill kernel reaches (the
// automatic choice up to 64 tokens is the decode kernel); it runs 64-token tiles (the
// template also builds 128 and 256):
//
// * The product is computed transposed, Y^T = W^T . X^T, so that the weights
//   are the MMA's A operand (M = 128 weight columns per CTA) and the tokens are
//   its N dimension.  A comes from tensor memory: dequantisation warps unpack
//   each int32 word (eight consecutive k of one column) into four 32-bit TMEM
//   cells of that column's lane, so dequantised weights never touch shared
//   memory.
// * Producer threads stream, per 64-k stage, the X tile [BT tokens x 64 k]
//   (FP16, 128-byte swizzle: the B operand), the qweight tile [8 packed rows x
//   128 columns] and the scale rows of the stage; out-of-range rows and
//   columns read as zero.
// * One thread issues tcgen05.mma (kind::f16, FP32 accumulate) into a
//   128 x BT FP32 accumulator in TMEM; tcgen05.commit releases each stage.
// * The dequantisation warps then read the accumulator back (tcgen05.ld),
//   round to FP16 and store Y.
// * Every wait is bounded in time; on expiry the kernel records
//   GPTQ_ERR_TIMEOUT in the device error word, drains its own copies and MMAs,
//   frees TMEM and exits.  Nothing traps.
//
// FLOPs per call: 2 M K N.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc05.cuh"
#include "tmap.h"

namespace gptq {

namespace {

constexpr int BW = 128;  // weight columns per CTA (MMA M; one TMEM lane each)
constexpr int BT_MAX = 256;  // tokens per CTA (MMA N): 64 in use, up to 256
constexpr int BK = 64;   // k per pipeline stage (four k16 MMAs)
constexpr int XS = 4;        // X ring stages (BT x 64 k each)
constexpr int WS = 8;        // weight-tile ring stages (qweight + scales of 64 k)
constexpr int AS = 8;        // A slots in TMEM (64 k each)
constexpr int DQ_GROUPS = 4;                // dequantisation groups, taking stages kb = g mod 4
constexpr int DQ_WARPS = 4 * DQ_GROUPS;     // one warp per TMEM lane quarter in each group
constexpr int DQ_WARP0 = 3;  // warps 0, 1, 2: X producer, MMA issuer, weight producer
constexpr int THREADS = (DQ_WARP0 + DQ_WARPS) * 32;
constexpr int QW_STAGE_BYTES = BW * (BK / 8) * 4;  // 128 columns x 8 packed rows: 4 KB
constexpr int S_ROW_BYTES = BW * 2;                // one scale row of the tile: 256 B
constexpr int S_STAGE_MAX_ROWS = BK / 16;          // group 16: four rows per stage
constexpr int W_STAGE_BYTES = QW_STAGE_BYTES + S_STAGE_MAX_ROWS * S_ROW_BYTES;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t D_COL = 0;                 // accumulator: columns [0, BT)
constexpr uint32_t A_COL = 256;               // A slots: [256, 256 + 8 * 32)
constexpr uint32_t A_STAGE_COLS = BK / 2;     // two FP16 per 32-bit column
constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr uint64_t kDrainLimitNs = 200000000ull;
static_assert(BT_MAX <= A_COL, "accumulator below the A slots");
static_assert(A_COL + AS * A_STAGE_COLS <= TMEM_COLS, "TMEM budget");
static_assert(AS == WS, "a weight stage and its A slot share an index");

// Shared-memory layout for a token tile of BT: the X ring, then the weight
// ring (qweight then scale rows per stage), then the barriers.
template <int BT>
struct Layout {
  static constexpr int X_STAGE_BYTES = BT * BK * 2;
  static constexpr int W_OFF = XS * X_STAGE_BYTES;
  static constexpr int BAR_OFF = W_OFF + WS * W_STAGE_BYTES;
  static constexpr size_t kSmemBytes = 1024 + (size_t)BAR_OFF + 512;
};

struct Barriers {
  uint64_t xfull[XS];    // X tile landed (TMA transaction count)
  uint64_t xempty[XS];   // MMAs reading the X tile done
  uint64_t wfull[WS];    // qweight and scale tiles landed
  uint64_t wempty[WS];   // weight tiles read by every dequantisation warp
  uint64_t afull[AS];    // A slot written by every dequantisation thread
  uint64_t aempty[AS];   // MMAs reading the A slot done
  uint64_t dfull;        // all MMAs of the tile done
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Barriers) <= 512, "barrier area");

// scale_rows: scale rows one 64-k stage touches (1, or 64/group for groups
// below 64); stages start on 64-k boundaries, so they align with groups.
//
// The X tiles and the weight tiles travel in separate rings: the weight ring
// and the A slots are twice as deep as the X ring, so the dequantisation runs
// up to eight stages ahead of the MMAs while the large X tiles only need four.
// A stage gives each dequantisation thread little work, so four groups of
// four warps take stages in turn (kb = g mod 4) and keep four stages in
// flight.
template <int BT>
__global__ void __launch_bounds__(THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap x_map,
                   const __grid_constant__ CUtensorMap qw_map,
                   const __grid_constant__ CUtensorMap s_map, uint16_t* __restrict__ y, int M,
                   int K, int N, int group_shift, int scale_rows, int* err) {
  static_assert(BT >= 64 && BT <= BT_MAX && BT % 64 == 0, "token tile");
  constexpr int X_STAGE_BYTES = Layout<BT>::X_STAGE_BYTES;
  constexpr int W_OFF = Layout<BT>::W_OFF;
  constexpr int BAR_OFF = Layout<BT>::BAR_OFF;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array itself so that the
  // compiler keeps the shared address space (plain LDS, no generic loads)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* xs = smem;
  Barriers* bar = reinterpret_cast<Barriers*>(smem + BAR_OFF);
  volatile int* abort_flag = &bar->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BW;
  const int t0 = blockIdx.y * BT;
  const int KB = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < XS; ++s) {
      mbar_init(&bar->xfull[s], 1);
      mbar_init(&bar->xempty[s], 1);
    }
    for (int j = 0; j < WS; ++j) {
      mbar_init(&bar->wfull[j], 1);
      mbar_init(&bar->wempty[j], 4);        // the four warps of the stage's group
      mbar_init(&bar->afull[j], 4 * 32);    // every thread of that group
      mbar_init(&bar->aempty[j], 1);
    }
    mbar_init(&bar->dfull, 1);
    bar->abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&x_map);
    prefetch_tensormap(&qw_map);
    prefetch_tensormap(&s_map);
  }
  if (warp == 1) {
    tmem_alloc(&bar->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 0 || warp == 2) {
    // ---------------- TMA producers: X (warp 0), weights (warp 2) ----------------
    if (lane == 0) {
      const bool xp = warp == 0;
      const int depth = xp ? XS : WS;
      int issued = 0;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % depth;
        const uint32_t ph = (uint32_t)(kb / depth) & 1u;
        uint64_t* emp = xp ? &bar->xempty[s] : &bar->wempty[s];
        if (!mbar_wait_bounded(emp, ph ^ 1u, abort_flag, kWaitLimitNs)) {
          record_timeout(err, bar);
          break;
        }
        if (xp) {
          mbar_arrive_expect_tx(&bar->xfull[s], X_STAGE_BYTES);
          tma_load_2d(xs + s * X_STAGE_BYTES, &x_map, kb * BK, t0, &bar->xfull[s]);
        } else {
          uint8_t* wst = smem + W_OFF + s * W_STAGE_BYTES;
          mbar_arrive_expect_tx(&bar->wfull[s], QW_STAGE_BYTES + scale_rows * S_ROW_BYTES);
          tma_load_2d(wst, &qw_map, n0, kb * (BK / 8), &bar->wfull[s]);
          tma_load_2d(wst + QW_STAGE_BYTES, &s_map, n0, (int)(((int64_t)kb * BK) >> group_shift),
                      &bar->wfull[s]);
        }
        ++issued;
      }
      if (*abort_flag) {
        // drain: wait for the last load issued into each slot
        int never = 0;
        for (int j = issued - 1; j >= 0 && j >= issued - depth; --j)
          mbar_wait_bounded(xp ? &bar->xfull[j % depth] : &bar->wfull[j % depth],
                            (uint32_t)(j / depth) & 1u, &never, kDrainLimitNs);
      }
    }
    __syncwarp();  // the whole warp reaches the CTA barrier below together
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // The whole warp runs the loop converged (so the descriptors stay
    // warp-uniform) and one elected lane issues the MMAs and commits.
    const uint32_t idesc = idesc_f16_f32(BW, BT);
    bool ok = true;
    for (int kb = 0; kb < KB && ok; ++kb) {
      const int s = kb % XS, a = kb % AS;
      ok = __all_sync(0xffffffffu,
                      mbar_wait_bounded(&bar->xfull[s], (uint32_t)(kb / XS) & 1u, abort_flag,
                                        kWaitLimitNs) &&
                          mbar_wait_bounded(&bar->afull[a], (uint32_t)(kb / AS) & 1u, abort_flag,
                                            kWaitLimitNs));
      if (!ok) break;
      tc_fence_after();
      const uint64_t b_desc0 = smem_desc_sw128(smem_u32(xs + s * X_STAGE_BYTES));
      const uint32_t a_base = tmem + A_COL + a * A_STAGE_COLS;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          mma_f16_ts(tmem + D_COL, a_base + kk * 8, b_desc0 + (uint64_t)((kk * 32) >> 4), idesc,
                     (kb | kk) != 0 ? 1u : 0u);
        mma_commit(&bar->xempty[s]);
        mma_commit(&bar->aempty[a]);
      }
      __syncwarp();
    }
    if (!ok && lane == 0) record_timeout(err, bar);
    if (elect_one()) mma_commit(&bar->dfull);
    __syncwarp();
    if (!ok) {
      int never = 0;
      mbar_wait_bounded(&bar->dfull, 0, &never, kDrainLimitNs);
    }
    __syncwarp();  // the whole warp reaches the CTA barrier below together
  } else {
    // ---------------- dequantisation, then epilogue ----------------
    const int quarter = warp & 3;                 // TMEM lanes 32*quarter .. +31
    const int grp = (warp - DQ_WARP0) >> 2;       // stages kb = grp mod DQ_GROUPS
    const int n = n0 + 32 * quarter + lane;
    const bool col_ok = n < N;
    const uint32_t lane_addr = (uint32_t)(32 * quarter) << 16;

    // this thread's column in the stage's qweight and scale tiles: all eight
    // packed rows of its group's stages
    const int col = 32 * quarter + lane;
    const uint8_t* qw_tile = smem + W_OFF + col * 4;
    const uint8_t* s_tile = smem + W_OFF + QW_STAGE_BYTES + col * 2;

    bool ok = true;
    for (int kb = grp; kb < KB; kb += DQ_GROUPS) {
      const int j = kb % WS;
      const uint32_t ph = (uint32_t)(kb / WS) & 1u;
      // qweight and scale tiles of the stage have landed
      ok = __all_sync(0xffffffffu,
                      mbar_wait_bounded<true>(&bar->wfull[j], ph, abort_flag, kWaitLimitNs));
      if (!ok) {
        if (lane == 0) record_timeout(err, bar);
        break;
      }
      const uint8_t* qw = qw_tile + j * W_STAGE_BYTES;
      const uint8_t* sc = s_tile + j * W_STAGE_BYTES;
      uint32_t cells[32];
#pragma unroll
      for (int r = 0; r < BK / 8; ++r) {
        // scale row of packed row r inside the stage (0 unless the group is
        // smaller than the 64-k stage)
        const int gl = (r * 8) >> group_shift;
        const uint16_t sv = *reinterpret_cast<const uint16_t*>(sc + gl * S_ROW_BYTES);
        const uint32_t w = *reinterpret_cast<const uint32_t*>(qw + r * (BW * 4));
        uint32_t nat[4];
        dequant_word_natural(w, half2_broadcast(sv), nat);
#pragma unroll
        for (int q = 0; q < 4; ++q) cells[4 * r + q] = nat[q];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->wempty[j]);  // weight tiles of the stage read
      // the A slot is free once the MMAs of its previous use have completed
      ok = __all_sync(0xffffffffu, mbar_wait_bounded<true>(&bar->aempty[j], ph ^ 1u, abort_flag,
                                                           kWaitLimitNs));
      if (!ok) {
        if (lane == 0) record_timeout(err, bar);
        break;
      }
      tc_fence_after();
      tmem_st_32x32b_x32(tmem + lane_addr + A_COL + j * A_STAGE_COLS, cells);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar->afull[j]);
    }

    if (ok) {
      ok = mbar_wait_bounded<true>(&bar->dfull, 0, abort_flag, kWaitLimitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok && lane == 0) record_timeout(err, bar);
    }
    if (ok) {
      // group g writes tokens [g*BT/4, (g+1)*BT/4) of the tile, 16 at a time
      tc_fence_after();
      constexpr int TPG = BT / DQ_GROUPS;
#pragma unroll 1
      for (int chunk = 0; chunk < TPG / 16; ++chunk) {
        const int tok0 = TPG * grp + 16 * chunk;
        uint32_t r[16];
        tmem_ld_32x32b_x16(tmem + lane_addr + D_COL + tok0, r);
        tmem_wait_ld();
        if (col_ok) {
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int t = t0 + tok0 + q;
            if (t < M)
              y[(int64_t)t * N + n] = __half_as_ushort(__float2half_rn(__uint_as_float(r[q])));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Tensor maps and launch for a token tile of BT.
template <int BT>
cudaError_t launch_t(const uint16_t* x, const int32_t* qweight, const uint16_t* scales, uint16_t* y,
                     int64_t M, int64_t K, int64_t N, int group_shift, int scale_rows,
                     int64_t n_groups, cudaStream_t stream, const DeviceInfo& dev) {
  CUtensorMap x_map, qw_map, s_map;
  if (!tensor_map_2d(&x_map, x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)K, (uint64_t)M,
                     (uint64_t)K * 2, BK, BT, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tensor_map_2d(&qw_map, qweight, CU_TENSOR_MAP_DATA_TYPE_INT32, (uint64_t)N,
                     (uint64_t)(K / 8), (uint64_t)N * 4, BW, BK / 8, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !tensor_map_2d(&s_map, scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, (uint64_t)N,
                     (uint64_t)n_groups, (uint64_t)N * 2, BW, (uint32_t)scale_rows,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  constexpr size_t smem = Layout<BT>::kSmemBytes;
  static std::once_flag attr_once[64];
  static cudaError_t attr_err[64];
  const int d = dev.device & 63;
  std::call_once(attr_once[d], [&] {
    attr_err[d] = cudaFuncSetAttribute(prefill_kernel<BT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  });
  if (attr_err[d] != cudaSuccess) return attr_err[d];
  const dim3 grid((unsigned)((N + BW - 1) / BW), (unsigned)((M + BT - 1) / BT), 1);
  prefill_kernel<BT><<<grid, THREADS, smem, stream>>>(x_map, qw_map, s_map, y, (int)M, (int)K,
                                                      (int)N, group_shift, scale_rows,
                                                      dev.error_word);
  return cudaGetLastError();
}

}  // namespace

// Up to 32 tokens (reached only when prefill is forced: the dispatcher sends
// M <= 64 to the decode kernel) one CTA per 128 columns x 64 tokens; above
// that the pair kernel, whose token tile (128 or 256) follows M.
cudaError_t launch_prefill(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                           uint16_t* y, int64_t M, int64_t K, int64_t N, int group_shift,
                           cudaStream_t stream, const DeviceInfo& dev) {
  const int64_t n_groups = (group_shift == 62 || (int64_t(1) << group_shift) >= K)
                               ? 1 : (K + (int64_t(1) << group_shift) - 1) >> group_shift;
  const int scale_rows = group_shift >= 6 ? 1 : (BK >> group_shift);
  // above 32 tokens the persistent CTA-pair kernel takes over (128- or
  // 256-token pair tiles): half the X traffic per SM, no per-tile launch
  if (M > 32)
    return launch_prefill_pair(x, qweight, scales, y, M, K, N, group_shift, stream, dev);
  return launch_t<64>(x, qweight, scales, y, M, K, N, group_shift, scale_rows, n_groups, stream,
                      dev);
}

}  // namespace gptq
