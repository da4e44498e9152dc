// Prefill kernel: Y[M, N] = X[M, K] . dequant(qweight, scales) for any M,
// on the 5th-generation tensor cores (tcgen05) with TMEM accumulators.
//
// Operation: GPTQ-Pro README, "Runtime contract" and "Ampere kernel
// architecture" (tensor-core prefill with FP32 accumulation that reads the
// native int32 qweight; predicated tails; FP16 output).  The Ampere design
// (cp.async staging, mma.sync) is prior art only.  On sm_100a:
//
// * The product is computed transposed, Y^T = W^T . X^T, so that the weights
//   are the MMA's A operand (M = 128 weight columns per CTA) and the tokens are
//   its N dimension (256 per CTA).  A comes from tensor memory: dequantisation
//   warps unpack each int32 word (eight consecutive k of one column) into four
//   32-bit TMEM cells of that column's lane, so dequantised weights never
//   touch shared memory.
// * X is the B operand: a TMA producer warp streams [256 tokens x 64 k] FP16
//   tiles into shared memory with the 128-byte swizzle the MMA descriptor
//   expects; out-of-range tokens and k read as zero.
// * One thread issues tcgen05.mma (kind::f16, FP32 accumulate) into a
//   128 x 256 FP32 accumulator in TMEM; tcgen05.commit releases each stage.
// * The dequantisation warps then read the accumulator back (tcgen05.ld),
//   round to FP16 and store Y.
// * Every wait is bounded in time; on expiry the kernel records
//   GPTQ_ERR_TIMEOUT in the device error word, drains its own copies and MMAs,
//   frees TMEM and exits.  Nothing traps.
//
// Bytes per CTA tile: 128 x K / 2 (qweight) + scales + 256 x K x 2 (X, from L2).
// FLOPs per call: 2 M K N.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc05.cuh"

namespace gptq {

namespace {

constexpr int BW = 128;  // weight columns per CTA (MMA M; one TMEM lane each)
constexpr int BT = 256;  // tokens per CTA (MMA N)
constexpr int BK = 64;   // k per pipeline stage (four k16 MMAs)
constexpr int STAGES = 4;
constexpr int DQ_WARPS = 8;  // dequantisation + epilogue warps
constexpr int THREADS = (2 + DQ_WARPS) * 32;
constexpr int X_STAGE_BYTES = BT * BK * 2;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t D_COL = 0;                 // accumulator: columns [0, 256)
constexpr uint32_t A_COL = 256;               // A stages: [256, 256 + 4 * 32)
constexpr uint32_t A_STAGE_COLS = BK / 2;     // two FP16 per 32-bit column
constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr uint64_t kDrainLimitNs = 200000000ull;
constexpr size_t kSmemBytes = 1024 + (size_t)STAGES * X_STAGE_BYTES + 256;

struct Barriers {
  uint64_t xfull[STAGES];   // X tile landed (TMA transaction count)
  uint64_t afull[STAGES];   // A stage written by all dequantisation threads
  uint64_t empty[STAGES];   // MMAs of the stage done: X slot and A columns free
  uint64_t dfull;           // all MMAs of the tile done
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ void record_timeout(int* err, Barriers* b) {
  atomicExch(err, kDeviceErrTimeout);
  *reinterpret_cast<volatile int*>(&b->abort_flag) = 1;
}

__global__ void __launch_bounds__(THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap x_map, const int32_t* __restrict__ qweight,
                   const uint16_t* __restrict__ scales, uint16_t* __restrict__ y, int M, int K,
                   int N, int group_shift, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* xs = smem;
  Barriers* bar = reinterpret_cast<Barriers*>(smem + STAGES * X_STAGE_BYTES);
  volatile int* abort_flag = &bar->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BW;
  const int t0 = blockIdx.y * BT;
  const int KB = (K + BK - 1) / BK;
  const int P = K >> 3;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bar->xfull[s], 1);
      mbar_init(&bar->afull[s], DQ_WARPS * 32);
      mbar_init(&bar->empty[s], 1);
    }
    mbar_init(&bar->dfull, 1);
    bar->abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) prefetch_tensormap(&x_map);
  if (warp == 1) {
    tmem_alloc(&bar->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer (one lane) ----------------
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
        if (!mbar_wait_bounded(&bar->empty[s], ph ^ 1u, abort_flag, kWaitLimitNs)) {
          record_timeout(err, bar);
          break;
        }
        mbar_arrive_expect_tx(&bar->xfull[s], X_STAGE_BYTES);
        tma_load_2d(xs + s * X_STAGE_BYTES, &x_map, kb * BK, t0, &bar->xfull[s]);
        ++issued;
      }
      if (*abort_flag) {
        // drain: wait for the last load issued into each slot
        int never = 0;
        for (int j = issued - 1; j >= 0 && j >= issued - STAGES; --j)
          mbar_wait_bounded(&bar->xfull[j % STAGES], (uint32_t)(j / STAGES) & 1u, &never,
                            kDrainLimitNs);
      }
    }
    __syncwarp();  // the whole warp reaches the CTA barrier below together
  } else if (warp == 1) {
    // ---------------- MMA issuer (one lane) ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(BW, BT);
      bool aborted = false;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
        if (!mbar_wait_bounded(&bar->xfull[s], ph, abort_flag, kWaitLimitNs) ||
            !mbar_wait_bounded(&bar->afull[s], ph, abort_flag, kWaitLimitNs)) {
          record_timeout(err, bar);
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint32_t xa = smem_u32(xs + s * X_STAGE_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint32_t a_tmem = tmem + A_COL + s * A_STAGE_COLS + kk * 8;
          const uint64_t b_desc = smem_desc_sw128(xa + kk * 32);
          mma_f16_ts(tmem + D_COL, a_tmem, b_desc, idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        mma_commit(&bar->empty[s]);
      }
      mma_commit(&bar->dfull);
      if (aborted) {
        int never = 0;
        mbar_wait_bounded(&bar->dfull, 0, &never, kDrainLimitNs);
      }
    }
    __syncwarp();  // the whole warp reaches the CTA barrier below together
  } else {
    // ---------------- dequantisation, then epilogue ----------------
    const int quarter = warp & 3;          // TMEM lanes 32*quarter .. +31
    const int half = (warp - 2) >> 2;      // packed rows 4*half .. +3 of a stage
    const int n = n0 + 32 * quarter + lane;
    const bool col_ok = n < N;
    const uint32_t lane_addr = (uint32_t)(32 * quarter) << 16;

    uint32_t cw[4], cs[4], nw[4], ns[4];
    auto load = [&](int kb, uint32_t (&w)[4], uint32_t (&sc)[4]) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int row = kb * (BK / 8) + 4 * half + r;
        if (col_ok && row < P) {
          w[r] = ld_nc_u32(qweight + (int64_t)row * N + n);
          sc[r] = ld_nc_u16(scales + ((int64_t(row) * 8) >> group_shift) * N + n);
        } else {
          w[r] = 0x88888888u;  // every code 8: weight (8 - 8) * 0 = 0
          sc[r] = 0;
        }
      }
    };

    bool ok = true;
    load(0, cw, cs);
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
      if (kb + 1 < KB) load(kb + 1, nw, ns);
      uint32_t cells[16];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        uint32_t nat[4];
        dequant_word_natural(cw[r], half2_broadcast((uint16_t)cs[r]), nat);
#pragma unroll
        for (int j = 0; j < 4; ++j) cells[4 * r + j] = nat[j];
      }
      ok = mbar_wait_bounded(&bar->empty[s], ph ^ 1u, abort_flag, kWaitLimitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) record_timeout(err, bar);
        break;
      }
      tc_fence_after();
      tmem_st_32x32b_x16(tmem + lane_addr + A_COL + s * A_STAGE_COLS + 16 * half, cells);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar->afull[s]);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        cw[r] = nw[r];
        cs[r] = ns[r];
      }
    }

    if (ok) {
      ok = mbar_wait_bounded(&bar->dfull, 0, abort_flag, kWaitLimitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok && lane == 0) record_timeout(err, bar);
    }
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int chunk = 0; chunk < (BT / 2) / 32; ++chunk) {
        const int tok0 = (BT / 2) * half + 32 * chunk;
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + lane_addr + D_COL + tok0, r);
        tmem_wait_ld();
        if (col_ok) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int t = t0 + tok0 + j;
            if (t < M)
              y[(int64_t)t * N + n] = __half_as_ushort(__float2half_rn(__uint_as_float(r[j])));
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

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

cudaError_t launch_prefill(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                           uint16_t* y, int64_t M, int64_t K, int64_t N, int group_shift,
                           cudaStream_t stream, const DeviceInfo& dev) {
  EncodeTiledFn encode = get_encode_fn();
  if (!encode) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
  const cuuint64_t gstride[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {BK, BT};
  const cuuint32_t estride[2] = {1, 1};
  if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(x), gdim, gstride,
             box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  static std::once_flag attr_once[64];
  static cudaError_t attr_err[64];
  const int d = dev.device & 63;
  std::call_once(attr_once[d], [&] {
    attr_err[d] = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  });
  if (attr_err[d] != cudaSuccess) return attr_err[d];
  const dim3 grid((unsigned)((N + BW - 1) / BW), (unsigned)((M + BT - 1) / BT), 1);
  prefill_kernel<<<grid, THREADS, kSmemBytes, stream>>>(map, qweight, scales, y, (int)M, (int)K,
                                                       (int)N, group_shift, dev.error_word);
  return cudaGetLastError();
}

}  // namespace gptq
