// Decode kernel: Y[M, N] = X[M, K] . dequant(qweight, scales) for M <= 64,
// on the 5th-generation tensor cores (tcgen05) with TMEM accumulators.
//
// Operation: GPTQ-Pro README, "Runtime contract" and "Ampere kernel
// architecture" (fused small-M decode that reads the native int32 qweight,
// keeps scales resident, and reduces split-K partial sums deterministically).
// The Ampere design (four-warp output tiles, warp-level MMA, M <= 4) is prior
// art only.  On sm_100a the warp-level mma.sync path cannot keep up with the
// weight stream, so this kernel is laid out around tcgen05:
//
// * The product is computed transposed, Y^T = W^T . X^T: a CTA owns 128 weight
//   columns (the MMA's M, one TMEM lane each) and a range of K; the tokens are
//   the MMA's N = BT, 16, 32, 48 or 64 (rows at or beyond M read as zero).
// * One TMA producer thread streams, per stage of 512 or 256 k, the qweight
//   tile [64 or 32 packed rows x 128 columns] (32 or 16 KB), the scale rows of
//   the stage and the X tile [BT tokens x the stage's k] (FP16, 128-byte
//   swizzle: the B operand; one 3-D box when K is a multiple of 64) into a
//   ring of stages in shared memory (224 KB: two to eight stages, depending
//   on BT and the stage's k).  512-k stages serve the 16-token tile when a
//   CTA streams the whole K of its columns, and adapters; 256-k stages
//   everything else (a split K range, or a token tile whose X leaves room for
//   only two or three 512-k stages).
// * Sixteen dequantisation warps in two groups of eight take alternate stages
//   (so one group's waits overlap the other's arithmetic); in a group, two
//   k-slices x four TMEM lane quarters each turn eight words of their column
//   at a time into 32 TMEM cells of an A slot (256 k per slot, three slots).
//   A word's codes come out paired (k, k+4) from the magic-number unpack;
//   rather than shuffling every weight back to natural order, the same warps
//   permute the (few) X rows of the stage in place to the paired order, so A
//   and B agree on the order of k inside every 8-k block.
// * Each weight is dequantised exactly as defined, fp16((q - 8) * s): 1024 + q
//   by a LOP3 into the FP16 mantissa of 1024, minus 1032 (exact), times the
//   group scale (one rounding).  Keeping the definition's per-weight rounding
//   matters: on inputs with large activation outliers, skipping it (scaling
//   FP32 partial sums per group instead) moves Y by up to ~1e-2 relative.
// * One elected lane of a converged MMA warp issues tcgen05.mma (kind::f16,
//   A from TMEM, B from shared memory, FP32 accumulate in TMEM);
//   tcgen05.commit releases the A slot of each fill and the ring slot of each
//   stage.  With only 16 tokens an MMA is short, and MMAs
//   into one accumulator run one after another, so the k16 steps go round-robin
//   to NACC independent accumulators, summed in a fixed order at the end.
// * Split-K: the `splits` CTAs of a thread-block cluster take consecutive K
//   ranges of the same columns and are reduced in a fixed order through
//   distributed shared memory: bitwise reproducible, no global scratch.
// * Programmatic dependent launch: before waiting for the previous kernel in
//   the stream, the producer only prefetches its first weight tiles into L2 (a
//   prefetch cannot observe stale data); every copy into shared memory and
//   every store of Y happens after the wait.  With a LoRA adapter the previous
//   launch is the one computing T, which is launched without this attribute
//   (it starts after all earlier work completed): then only the first read of
//   T waits, and the K stages overlap that launch.  Once it has issued its
//   last copy, the producer lets the next kernel in the stream begin its
//   prologue.
// * Every wait is bounded in time; on expiry the kernel records
//   GPTQ_ERR_TIMEOUT in the device error word, drains its own copies and MMAs,
//   frees TMEM and exits.  Nothing traps.
//
// Bytes per call: K*N/2 (qweight) + n_groups*N*2 (scales) + M*K*2 + M*N*2.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "gptq_w4a16.h"
#include "kernels.h"
#include "tc05.cuh"
#include "tmap.h"

namespace gptq {

namespace {

constexpr int BW = 128;                  // weight columns per CTA (MMA M)
constexpr int BKA = 256;                 // k per A slot fill (16 MMAs of k16)
constexpr int PRA = BKA / 8;             // packed rows per A slot fill
constexpr int GROUPS = 2;                // dequantisation groups, taking alternate stages
constexpr int SLICES = 2;                // k slices of an A slot fill within a group
constexpr int WPT = 8;                   // words per TMEM store (32 columns)
constexpr int CHUNKS = PRA / (SLICES * WPT);  // TMEM stores per thread per fill
constexpr int GROUP_WARPS = 4 * SLICES;  // four TMEM lane quarters per slice
constexpr int DQ_WARPS = GROUPS * GROUP_WARPS;
constexpr int THREADS = (2 + DQ_WARPS) * 32;
// A LoRA stage's lora_b tile: 128 rows x 64 ranks (128-byte rows, 128-byte
// swizzle) per half, two halves in the qweight area.
constexpr int LORA_HALF_BYTES = BW * 64 * 2;
constexpr int S_ROW_BYTES = BW * 2;
constexpr int Z_ROW_BYTES = BW / 8 * 4;  // one row of packed zero points (asymmetric weights)
constexpr int kMaxStages = 8;
constexpr int kRingBudget = 224 * 1024;
constexpr int A_SLOTS = 3;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t D_COL = 0;            // accumulators: NACC x BT columns
constexpr uint32_t A_COL0 = 128;         // A slots: [128, 512), 128 columns each
constexpr uint32_t A_SLOT_COLS = BKA / 2;  // two FP16 per 32-bit column
constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr uint64_t kDrainLimitNs = 200000000ull;

static_assert(A_COL0 + A_SLOTS * A_SLOT_COLS <= TMEM_COLS, "TMEM budget");

// Geometry that depends on the token tile BT (the MMA's N) and on the packed
// rows per ring stage PRS (64: 512 k, two A slot fills; 32: 256 k, one
// fill): a stage holds X as X_ATOMS atoms of [BT tokens x 64 k] (128-byte
// swizzle), then qweight, then the scale rows.
template <int BT_, int PRS_>
struct TokGeo {
  static constexpr int BT = BT_;
  static constexpr int PRS = PRS_;                   // packed rows per ring stage
  static constexpr int BKS = 8 * PRS;                // k per ring stage
  static constexpr int HALVES = BKS / BKA;           // A slot fills per ring stage
  static constexpr int X_ATOMS = BKS / 64;
  static constexpr int QW_STAGE_BYTES = PRS * BW * 4;
  // adapter stages need room for two lora_b halves in the qweight area
  static constexpr bool LORA_OK = 2 * LORA_HALF_BYTES <= QW_STAGE_BYTES;
  static constexpr int X_ATOM_BYTES = BT * 128;
  static constexpr int X_STAGE_BYTES = X_ATOMS * X_ATOM_BYTES;
  static constexpr int QW_OFF = X_STAGE_BYTES;
  static constexpr int S_OFF = QW_OFF + QW_STAGE_BYTES;
  // independent accumulators (the k16 steps go round-robin), NACC x BT <= 128
  static constexpr int NACC = 128 / BT < 4 ? 128 / BT : 4;
  static_assert(BT % 16 == 0 && BT >= 16 && BT <= 64, "token tile");
  static_assert(PRS == PRA || PRS == 2 * PRA, "a stage is one or two A slot fills");
  static_assert(D_COL + NACC * BT <= A_COL0, "accumulators below the A slots");
  static_assert(BT * BW * 4 <= X_STAGE_BYTES + QW_STAGE_BYTES, "reduction buffer fits a stage");
};
static_assert(1024 + kRingBudget + 256 <= 227 * 1024, "shared memory per CTA");

struct DecodeShape {
  int scale_rows;   // scale rows per stage (the scale box height)
  int stage_bytes;  // X + qweight + scales of one stage (1024-aligned)
  int stages;       // ring depth
  int smem_bytes;   // whole dynamic allocation
  // act order: the resident scale tile and the token tiles of the grid
  int n_groups = 0;
  int tile_bytes = 0;
  int tile_boxes = 0;
  int tile_box_rows = 0;
  int tok_tiles = 1;
};

inline int align1024(int v) { return (v + 1023) & ~1023; }

// Stages start on multiples of their k extent BKS (512 or 256) and groups
// are powers of two, so a stage touches BKS / group scale rows (one for
// groups of BKS and more).
// With zero points (asym) each stage also holds their rows after the scales.
template <int BT, int PRS>
inline DecodeShape decode_shape(int group_shift, bool asym = false) {
  DecodeShape d;
  constexpr int BKS = TokGeo<BT, PRS>::BKS;
  const int gs = group_shift < 30 ? group_shift : 30;  // group -1 has shift 62
  d.scale_rows = (BKS >> gs) > 1 ? (BKS >> gs) : 1;
  d.stage_bytes = align1024(TokGeo<BT, PRS>::S_OFF +
                            d.scale_rows * (S_ROW_BYTES + (asym ? Z_ROW_BYTES : 0)));
  const int s = kRingBudget / d.stage_bytes;
  d.stages = s > kMaxStages ? kMaxStages : s;
  d.smem_bytes = 1024 + d.stages * d.stage_bytes + 256;
  return d;
}

// Act order: the scale tile of every group in front of the ring, loaded as
// the fewest boxes of at most 256 rows; each stage carries its BKS entries of
// g_idx in place of scale rows.
template <int BT, int PRS>
inline DecodeShape decode_shape_gidx(int64_t n_groups) {
  using G = TokGeo<BT, PRS>;
  DecodeShape d;
  d.scale_rows = 0;
  d.n_groups = (int)n_groups;
  d.tile_boxes = (int)((n_groups + 255) / 256);
  d.tile_box_rows = (int)((n_groups + d.tile_boxes - 1) / d.tile_boxes);
  d.tile_bytes = align1024(d.tile_boxes * d.tile_box_rows * S_ROW_BYTES);
  d.stage_bytes = align1024(G::S_OFF + G::BKS * 4);
  const int s = d.tile_bytes < kRingBudget ? (kRingBudget - d.tile_bytes) / d.stage_bytes : 0;
  d.stages = s > kMaxStages ? kMaxStages : s;
  d.smem_bytes = 1024 + d.tile_bytes + d.stages * d.stage_bytes + 256;
  return d;
}

struct DecodeBars {
  uint64_t full[kMaxStages];   // stage landed (TMA transaction count)
  uint64_t empty[kMaxStages];  // stage read by every dequantisation warp and the MMAs
  uint64_t afull[A_SLOTS];     // A slot written (and X permuted) by every dequantisation thread
  uint64_t aempty[A_SLOTS];    // MMAs reading the A slot done
  uint64_t dfull;              // all MMAs done
  uint64_t tile_full;          // act order: the CTA's scale tile landed
  uint64_t dblk[2];            // persistent: MMAs of a column block done (set j % 2)
  uint64_t dempty[2];          // persistent: accumulator set read out
  uint32_t tmem_base;
  int abort_flag;
};

constexpr int kMaxLinears = GPTQ_MAX_GROUPED;

// The linears of one launch: one for a plain call, several that share X for
// a grouped call.  Per linear its tensor maps, output and width, and the first
// column block of the grid that it owns (blk0[count] = total blocks).
struct LinearSet {
  CUtensorMap qw[kMaxLinears];
  CUtensorMap sc[kMaxLinears];
  uint16_t* y[kMaxLinears];
  int n[kMaxLinears];
  int blk0[kMaxLinears + 1];
  int count;
};

__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* map, int32_t c0, int32_t c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1)
               : "memory");
}

// One 16-byte chunk of an X row (eight consecutive k) rewritten in place from
// natural order (x0 .. x7) to the paired order of the unpacked weights:
// (x0, x4), (x1, x5), (x2, x6), (x3, x7).
__device__ __forceinline__ void permute_x_chunk(uint8_t* p) {
  uint4 v = *reinterpret_cast<const uint4*>(p);
  uint4 o;
  o.x = prmt(v.x, v.z, 0x5410);
  o.y = prmt(v.x, v.z, 0x7632);
  o.z = prmt(v.y, v.w, 0x5410);
  o.w = prmt(v.y, v.w, 0x7632);
  *reinterpret_cast<uint4*>(p) = o;
}

// The LoRA adapter's T computed by CTAs of the layer's own launch (the fused
// form, up to 32 tokens): `ctas` CTAs appended to the grid's column blocks
// (blockIdx.y == 0 of each computes; the others of its cluster only exit)
// each compute T for a balanced share of the ranks over all of K, store it,
// and add one to the low half of this call's hand-over slot.  Each of the
// `consumers` CTAs that run adapter stages waits for that count to reach
// `ctas` before its first read of T, then adds one to the high half; the last
// of them clears the slot, so that the slot starts at zero for its next use
// (the next call given it, or the same call replayed from a CUDA graph).
// ctas == 0: T comes from the launch before this one.
struct LoraFused {
  const uint16_t* x;           // X [M, K]
  const uint16_t* a;           // lora_a [rank, K]
  uint16_t* t;                 // T [M, rank]
  unsigned long long* flag;    // this call's slot
  int ctas;
  int consumers;
  int rank;
};

__device__ __forceinline__ unsigned long long ld_acquire_gpu_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Global-memory writes that this thread has observed (through an acquire)
// become visible to its later TMA reads.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Waits until the low half of *flag reaches `count`; false after limit_ns or
// once *abort is set.
__device__ __forceinline__ bool flag_wait_bounded(const unsigned long long* flag, uint32_t count,
                                                  volatile int* abort, uint64_t limit_ns) {
  if ((uint32_t)ld_acquire_gpu_u64(flag) >= count) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t n = 1;; ++n) {
    if ((uint32_t)ld_acquire_gpu_u64(flag) >= count) return true;
    if ((n & 63u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) return false;
    }
  }
}

// One CTA of the fused form: T[m, j] = fp16(sum_k X[m, k] lora_a[j, k]) for
// its ranks j (i-th of `ctas` balanced shares) and every token m < M <= MB.
// The ranks take the CTA's warps in equal groups that split K (a warp per
// rank, several ranks in turn, when there are more ranks than warps); lane l
// takes 8-k chunk l of every 256-k piece of its warp's range, X read in
// rounds of eight tokens.  FP32 sums in a fixed order: the lanes by shuffles,
// then the rank's warps in order.  X and lora_a are read with plain global
// loads after the grid-dependency wait (not through the read-only path: this
// grid may start while the previous one still runs).
template <int MB>
__device__ void lora_t_cta(const LoraFused& lf, int M, int K, int i, float* part) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // X may come from the previous kernel
  constexpr int NW = THREADS / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = (int)((int64_t)i * lf.rank / lf.ctas);
  const int nr = (int)((int64_t)(i + 1) * lf.rank / lf.ctas) - r0;
  const int wpr = nr > 0 && nr < NW ? NW / nr : 1;  // warps per rank
  const int ws = warp % wpr;                        // this warp's slice of K
  const int pieces = (K + 255) / 256;
  const int pb = ws * pieces / wpr, pe = (ws + 1) * pieces / wpr;
  for (int rr = warp / wpr; rr < nr; rr += NW / wpr) {
    float acc[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) acc[m] = 0.f;
    const uint16_t* arow = lf.a + (int64_t)(r0 + rr) * K;
    for (int pc = pb; pc < pe; ++pc) {
      const int k = pc * 256 + 8 * lane;
      if (k < K) {  // K % 8 == 0: the chunk is whole
        const uint4 av = *reinterpret_cast<const uint4*>(arow + k);
        const float2 a0 = __half22float2(*reinterpret_cast<const __half2*>(&av.x));
        const float2 a1 = __half22float2(*reinterpret_cast<const __half2*>(&av.y));
        const float2 a2 = __half22float2(*reinterpret_cast<const __half2*>(&av.z));
        const float2 a3 = __half22float2(*reinterpret_cast<const __half2*>(&av.w));
#pragma unroll
        for (int m0 = 0; m0 < MB; m0 += 8) {
          if (m0 >= M) break;
          uint4 xv[8];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            xv[q] = m0 + q < M ? *reinterpret_cast<const uint4*>(lf.x + (int64_t)(m0 + q) * K + k)
                               : make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int q = 0; q < 8; ++q) fma8(acc[m0 + q], xv[q], a0, a1, a2, a3);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      float v = acc[m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
      if (lane == 0) part[(rr * wpr + ws) * MB + m] = v;
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < nr * M; idx += THREADS) {
    const int rr = idx / M, m = idx - rr * M;
    float sum = 0.f;
    for (int w = 0; w < wpr; ++w) sum += part[(rr * wpr + w) * MB + m];
    lf.t[(int64_t)m * lf.rank + r0 + rr] = __half_as_ushort(__float2half_rn(sum));
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // every thread's stores of T, then this CTA's count (release at GPU scope)
    __threadfence();
    atomicAdd(lf.flag, 1ull);
  }
}

// WPS: consecutive words of a thread (8 k each) that share one scale: 2 for
// group 16, 4 for group 32, 8 (the thread's whole slice) for 64 and more.
// x3d: X arrives as one 3-D box per stage (K a multiple of 64) instead of
// one 2-D box per 64-k atom.
// ASYM: asymmetric weights (one linear): qz_map describes the packed zero
// points [n_groups, N/8]; each stage holds their rows after the scales and
// every column's zero replaces the 8 of the symmetric layer.
// lora_rank > 0: a LoRA adapter (one linear; GPTQ-Pro README, "Runtime
// contract": adapters on the linear path).  t_map describes T = fp16(X .
// lora_a^T) [M, rank] and b_map lora_b [N, rank].  The last CTA of each
// column block's split runs rank/128 more stages after its K stages: lora_b's
// 128 rows x 128 ranks go to the qweight area (two 64-rank boxes, 128-byte
// swizzle), T's rows to the X area (two 64-rank atoms); one fill per stage
// copies lora_b into the A slot in the paired k order (T is permuted like X),
// and the MMAs add T . lora_b^T to the same accumulators.  lf.ctas > 0 (the
// fused form, LoraFused above): the CTAs past the column blocks compute T,
// and the producer's first read of T waits on the hand-over counter instead
// of the grid dependency.
// GIDX (act order): every k has its own group g_idx[k].  The CTA's whole
// scale tile [n_groups x 128 columns] is loaded once into shared memory in
// front of the ring (tile_boxes boxes of tile_box_rows rows, tile_bytes in
// all; s_map's box is that high); each stage carries its slice of g_idx (in
// place of scale rows, through qz_map) and the dequantisation gathers one
// scale per k from the tile.  Token tiles: blockIdx.z takes tokens
// BT * blockIdx.z onwards (more than one tile only for act order).
// PERSIST (16-token tile, no split, plain weights): a grid smaller than the
// column blocks; CTA c takes blocks c, c + gridDim.x, ... one after another
// through the same ring, its MMAs alternating between two accumulator sets so
// that block j is read out (by the four slice-0 warps of group 0, between
// their stages) while block j + 1 streams.
template <int WPS, int BT, int PRS_, bool ASYM, bool GIDX, bool PERSIST>
__global__ void __launch_bounds__(THREADS, 1)
    decode_kernel(const __grid_constant__ CUtensorMap x_map, const __grid_constant__ LinearSet ls,
                  const __grid_constant__ CUtensorMap qz_map,
                  const __grid_constant__ CUtensorMap t_map,
                  const __grid_constant__ CUtensorMap b_map, int M, int K, int group_shift,
                  int stages, int stage_bytes, int scale_rows, int x3d, int lora_rank,
                  int n_groups, int tile_bytes, int tile_boxes, int tile_box_rows,
                  const __grid_constant__ LoraFused lf, int* err) {
  static_assert(!(GIDX && ASYM), "act order with symmetric weights only");
  static_assert(!PERSIST || (!ASYM && !GIDX && 2 * TokGeo<BT, PRS_>::NACC * BT <= A_COL0),
                "persistent: plain weights, two accumulator sets below the A slots");
  constexpr int X_ATOM_BYTES = TokGeo<BT, PRS_>::X_ATOM_BYTES;
  constexpr int X_STAGE_BYTES = TokGeo<BT, PRS_>::X_STAGE_BYTES;
  constexpr int QW_OFF = TokGeo<BT, PRS_>::QW_OFF;
  constexpr int S_OFF = TokGeo<BT, PRS_>::S_OFF;
  constexpr int NACC = TokGeo<BT, PRS_>::NACC;
  constexpr int PRS = TokGeo<BT, PRS_>::PRS;
  constexpr int BKS = TokGeo<BT, PRS_>::BKS;
  constexpr int HALVES = TokGeo<BT, PRS_>::HALVES;
  constexpr int X_ATOMS = TokGeo<BT, PRS_>::X_ATOMS;
  constexpr int QW_STAGE_BYTES = TokGeo<BT, PRS_>::QW_STAGE_BYTES;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array itself so that the
  // compiler keeps the shared address space (plain LDS, no generic loads)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  if constexpr (!PERSIST && !GIDX && !ASYM && TokGeo<BT, PRS_>::LORA_OK) {
    // fused adapter form: the CTAs past the column blocks compute T
    if (lf.ctas > 0 && (int)blockIdx.x >= ls.blk0[ls.count]) {
      if (blockIdx.y == 0 && blockIdx.z == 0)
        lora_t_cta<BT>(lf, M, K, (int)blockIdx.x - ls.blk0[ls.count],
                       reinterpret_cast<float*>(smem));
      return;
    }
  }
  // act order: the scale tile, then the ring (tile_bytes is a multiple of 1024)
  uint8_t* ring = smem + (GIDX ? tile_bytes : 0);
  DecodeBars* bar = reinterpret_cast<DecodeBars*>(ring + stages * stage_bytes);
  volatile int* abort_flag = &bar->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's linear and column block
  int li = 0;
  while (li + 1 < ls.count && (int)blockIdx.x >= ls.blk0[li + 1]) ++li;
  const CUtensorMap* qw_map = &ls.qw[li];
  const CUtensorMap* s_map = &ls.sc[li];
  uint16_t* __restrict__ y = ls.y[li];
  const int N = ls.n[li];
  const int n0 = ((int)blockIdx.x - ls.blk0[li]) * BW;
  const int tok0 = (int)blockIdx.z * BT;      // this CTA's first token
  const int Mt = min(M - tok0, BT);           // its tokens (1 .. BT)
  const int NS = ((K >> 3) + PRS - 1) / PRS;  // stages over all of K
  const int splits = gridDim.y;
  const int st_begin = (int)((int64_t)blockIdx.y * NS / splits);
  const int st_end = (int)((int64_t)(blockIdx.y + 1) * NS / splits);
  const int n_st = st_end - st_begin;
  // LoRA stages of this CTA (the last of the column block's split), then all
  const int n_lora = (TokGeo<BT, PRS_>::LORA_OK && lora_rank > 0 && (int)blockIdx.y == splits - 1)
                         ? (lora_rank + 127) / 128 : 0;
  // persistent: this CTA's column blocks (PERSIST launches have no split and
  // no adapter, so each block is n_st stages)
  const int n_blk = PERSIST ? (ls.blk0[ls.count] - (int)blockIdx.x + (int)gridDim.x - 1) /
                                  (int)gridDim.x
                            : 1;
  const int n_tot = PERSIST ? n_blk * n_st : n_st + n_lora;
  const int gs = min(group_shift, 30);        // group -1 (shift 62): row 0 throughout
  const int z_off = S_OFF + scale_rows * S_ROW_BYTES;  // zero-point rows (ASYM)

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&bar->full[s], 1);
      mbar_init(&bar->empty[s], GROUP_WARPS + 1);  // the stage's group + the MMA commit
    }
    for (int a = 0; a < A_SLOTS; ++a) {
      mbar_init(&bar->afull[a], GROUP_WARPS * 32);
      mbar_init(&bar->aempty[a], 1);
    }
    mbar_init(&bar->dfull, 1);
    mbar_init(&bar->tile_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar->dblk[i], 1);
      mbar_init(&bar->dempty[i], 4);  // the four read-out warps
    }
    bar->abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&x_map);
    prefetch_tensormap(qw_map);
    prefetch_tensormap(s_map);
    if (ASYM) prefetch_tensormap(&qz_map);
    if (n_lora > 0) {
      prefetch_tensormap(&t_map);
      prefetch_tensormap(&b_map);
    }
    // L2 prefetch of the first stages' weight tiles: safe before the wait
    const int pf = min(n_st, 2);
    for (int t = 0; t < pf; ++t) tma_prefetch_l2_2d(qw_map, n0, (st_begin + t) * PRS);
  }
  if (warp == 1) {
    tmem_alloc(&bar->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  // Without an adapter, or with T computed in this launch, the previous
  // kernel in the stream may still be running and may write X: every thread
  // waits for it here.  With T from a separate launch, that launch started
  // only after all earlier work had completed, so X, the weights and Y are
  // safe now and only the producer's first read of T waits for it (below).
  if (lora_rank == 0 || lf.ctas > 0) grid_dependency_wait();

  if (warp == 0) {
    // ---------------- TMA producer (one lane) ----------------
    if (lane == 0) {
      int issued = 0;
      int s = 0;
      uint32_t ph = 0;
      bool t_waited = false;
      if constexpr (GIDX) {
        // the scale tile of this CTA's columns: every group
        mbar_arrive_expect_tx(&bar->tile_full,
                              (uint32_t)(tile_boxes * tile_box_rows * S_ROW_BYTES));
        for (int b = 0; b < tile_boxes; ++b)
          tma_load_2d(smem + b * tile_box_rows * S_ROW_BYTES, s_map, n0, b * tile_box_rows,
                      &bar->tile_full);
      }
      for (int t = 0; t < n_tot; ++t) {
        if (!mbar_wait_bounded(&bar->empty[s], ph ^ 1u, abort_flag, kWaitLimitNs)) {
          record_timeout(err, bar);
          break;
        }
        // the first two stages go out alone, so that they land before the
        // rest of the ring is requested (every CTA starts at once)
        if (t == 2 && !mbar_wait_bounded(&bar->full[0], 0u, abort_flag, kWaitLimitNs)) {
          record_timeout(err, bar);
          break;
        }
        uint8_t* st = ring + s * stage_bytes;
        if (!PERSIST && t >= n_st) {
          // LoRA stage: ranks 128 l .. 128 l + 127, as two 64-rank halves
          // (a half wholly past the rank is neither loaded nor multiplied)
          if (t == n_st) {
            if (lf.ctas > 0) {
              // T from this launch's T CTAs: all of them done, then visible to
              // TMA; the last CTA past this point clears the slot
              if (!flag_wait_bounded(lf.flag, (uint32_t)lf.ctas, abort_flag, kWaitLimitNs)) {
                record_timeout(err, bar);
                break;
              }
              fence_proxy_async_global();
              const unsigned long long seen = atomicAdd(lf.flag, 1ull << 32);
              if ((seen >> 32) == (unsigned long long)(lf.consumers - 1)) atomicExch(lf.flag, 0ull);
            } else {
              grid_dependency_wait();  // T is complete and visible
            }
            t_waited = true;
          }
          const int r0 = 128 * (t - n_st);
          const uint32_t halves = r0 + 64 < lora_rank ? 2u : 1u;
          mbar_arrive_expect_tx(&bar->full[s], halves * (LORA_HALF_BYTES + X_ATOM_BYTES));
          for (uint32_t h = 0; h < halves; ++h) {
            tma_load_2d(st + QW_OFF + h * LORA_HALF_BYTES, &b_map, r0 + 64 * (int)h, n0,
                        &bar->full[s]);
            tma_load_2d(st + h * X_ATOM_BYTES, &t_map, r0 + 64 * (int)h, tok0, &bar->full[s]);
          }
          ++issued;
          if (++s == stages) {
            s = 0;
            ph ^= 1u;
          }
          continue;
        }
        const int ts = PERSIST ? t % n_st : t;  // stage within the column block
        const CUtensorMap* qwm = qw_map;
        const CUtensorMap* scm = s_map;
        int nb0 = n0;
        if constexpr (PERSIST) {
          const int b = (int)blockIdx.x + (t / n_st) * (int)gridDim.x;
          int l = 0;
          while (l + 1 < ls.count && b >= ls.blk0[l + 1]) ++l;
          qwm = &ls.qw[l];
          scm = &ls.sc[l];
          nb0 = (b - ls.blk0[l]) * BW;
        }
        const int k0 = (st_begin + ts) * BKS;
        mbar_arrive_expect_tx(&bar->full[s],
                              X_STAGE_BYTES + QW_STAGE_BYTES +
                                  (GIDX ? BKS * 4
                                        : scale_rows * (S_ROW_BYTES + (ASYM ? Z_ROW_BYTES : 0))));
        tma_load_2d(st + QW_OFF, qwm, nb0, k0 >> 3, &bar->full[s]);
        if constexpr (GIDX) {
          // g_idx[k0 .. k0 + BKS) as [BKS / 16 rows x 16]
          tma_load_2d(st + S_OFF, &qz_map, 0, k0 >> 4, &bar->full[s]);
        } else {
          tma_load_2d(st + S_OFF, scm, nb0, k0 >> gs, &bar->full[s]);
          if (ASYM) tma_load_2d(st + z_off, &qz_map, n0 / 8, k0 >> gs, &bar->full[s]);
        }
        if (x3d) {
          tma_load_3d(st, &x_map, 0, tok0, k0 >> 6, &bar->full[s]);
        } else {
#pragma unroll 1
          for (int a = 0; a < X_ATOMS; ++a)
            tma_load_2d(st + a * X_ATOM_BYTES, &x_map, k0 + 64 * a, tok0, &bar->full[s]);
        }
        ++issued;
        if (++s == stages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (*abort_flag) {
        // drain: wait (bounded) for the last load issued into each slot
        int never = 0;
        for (int j = issued - 1; j >= 0 && j >= issued - stages; --j)
          mbar_wait_bounded(&bar->full[j % stages], (uint32_t)(j / stages) & 1u, &never,
                            kDrainLimitNs);
        if (GIDX) mbar_wait_bounded(&bar->tile_full, 0u, &never, kDrainLimitNs);
      }
      // a CTA with adapter stages completes only after the launch computing T
      // (so this grid's completion implies T's, also when it gave up early)
      if (n_lora > 0 && !t_waited) grid_dependency_wait();
      // all of this CTA's copies are issued: the next kernel in the stream may
      // start its prologue (it waits for this grid before touching its inputs)
      allow_dependent_launch();
    }
    __syncwarp();  // the whole warp reaches the CTA barrier below together
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // The whole warp runs the loop converged (so the descriptors stay
    // warp-uniform) and one elected lane issues the MMAs and commits.
    const uint32_t idesc = idesc_f16_f32(BW, BT);
    bool ok = true;
    int s = 0, a = 0;
    uint32_t ph = 0, aph = 0;
    for (int t = 0; t < n_tot && ok; ++t) {
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar->full[s], ph, abort_flag, kWaitLimitNs));
      const uint64_t x_desc = smem_desc_sw128(smem_u32(ring + s * stage_bytes));
      if constexpr (GIDX) {
        // every group index of the stage in range (the dequantisation clamps
        // them, so a bad one reads inside the tile; it is reported here)
        if (ok) {
          const uint32_t* gi = reinterpret_cast<const uint32_t*>(ring + s * stage_bytes + S_OFF);
          bool bad = false;
#pragma unroll 4
          for (int i = lane; i < BKS; i += 32) bad |= gi[i] >= (uint32_t)n_groups;
          if (__any_sync(0xffffffffu, bad) && lane == 0) atomicCAS(err, 0, kDeviceErrIndex);
        }
      }
      if (!PERSIST && t >= n_st) {
        // LoRA stage: one fill, one k16 step per 16 ranks of the stage
        if (ok)
          ok = __all_sync(0xffffffffu,
                          mbar_wait_bounded(&bar->afull[a], aph, abort_flag, kWaitLimitNs));
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_base = tmem + A_COL0 + a * A_SLOT_COLS;
        const int nk = min(128, lora_rank - 128 * (t - n_st)) / 16;
        if (elect_one()) {
          for (int kk = 0; kk < nk; ++kk)
            mma_f16_ts(tmem + D_COL + (kk % NACC) * BT, a_base + 8 * kk,
                       x_desc + (uint64_t)(((kk >> 2) * X_ATOM_BYTES + (kk & 3) * 32) >> 4),
                       idesc, 1u);
          mma_commit(&bar->aempty[a]);
          mma_commit(&bar->empty[s]);
        }
        __syncwarp();
        if (++a == A_SLOTS) {
          a = 0;
          aph ^= 1u;
        }
        if (++s == stages) {
          s = 0;
          ph ^= 1u;
        }
        continue;
      }
      // persistent: column block j of this CTA, stage ts of it, and its
      // accumulator set (free again once block j - 2 has been read out)
      const int j = PERSIST ? t / n_st : 0;
      const int ts = PERSIST ? t - j * n_st : t;
      const uint32_t d_base = tmem + D_COL + (uint32_t)((j & 1) * NACC * BT);
      if (PERSIST && ts == 0 && j >= 2) {
        if (ok)
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar->dempty[j & 1],
                                                         (uint32_t)((j - 2) >> 1) & 1u,
                                                         abort_flag, kWaitLimitNs));
        if (!ok) break;
        tc_fence_after();
      }
#pragma unroll
      for (int hf = 0; hf < HALVES; ++hf) {
        if (ok)
          ok = __all_sync(0xffffffffu,
                          mbar_wait_bounded(&bar->afull[a], aph, abort_flag, kWaitLimitNs));
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_base = tmem + A_COL0 + a * A_SLOT_COLS;
        // k16 step kk of this fill reads X atom 4*hf + kk/4 at byte (kk % 4) * 32
        // (the descriptor's address field counts 16 bytes)
        const uint64_t b_desc0 = x_desc + (uint64_t)((hf * 4 * X_ATOM_BYTES) >> 4);
        const uint32_t first = (ts == 0 && hf == 0) ? 0u : 1u;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < BKA / 16; ++kk)
            mma_f16_ts(d_base + (kk % NACC) * BT, a_base + 8 * kk,
                       b_desc0 + (uint64_t)(((kk >> 2) * X_ATOM_BYTES + (kk & 3) * 32) >> 4),
                       idesc, kk >= NACC ? 1u : first);
          mma_commit(&bar->aempty[a]);
          if (hf == HALVES - 1) mma_commit(&bar->empty[s]);
          if (PERSIST && hf == HALVES - 1 && ts == n_st - 1) mma_commit(&bar->dblk[j & 1]);
        }
        __syncwarp();
        if (++a == A_SLOTS) {
          a = 0;
          aph ^= 1u;
        }
      }
      if (++s == stages) {
        s = 0;
        ph ^= 1u;
      }
    }
    if (!ok && lane == 0) record_timeout(err, bar);
    if (elect_one()) mma_commit(&bar->dfull);
    __syncwarp();
    if (!ok) {
      // wait (bounded) for the MMAs already issued before freeing TMEM
      int never = 0;
      mbar_wait_bounded(&bar->dfull, 0, &never, kDrainLimitNs);
    }
    __syncwarp();  // the whole warp reaches the CTA barrier below together
  } else {
    // ---------------- dequantisation, then epilogue ----------------
    // Two groups of eight warps take alternate stages, so that one group's
    // waits overlap the other's arithmetic.  Within a group, slice hs of
    // quarter q dequantises packed rows 16*hs .. 16*hs+15 of each fill for
    // the columns of TMEM lanes 32q .. 32q+31, in two stores of eight words.
    const int dw = warp - 2;
    const int grp = dw / GROUP_WARPS;
    const int quarter = warp & 3;        // TMEM lanes 32*quarter .. +31
    const int hs = (dw % GROUP_WARPS) >> 2;
    const int h = dw >> 2;               // 0 only for the four epilogue warps
    const int col = 32 * quarter + lane;
    const int n = n0 + col;
    const uint32_t lane_addr = (uint32_t)(32 * quarter) << 16;
    const int gid = (dw % GROUP_WARPS) * 32 + lane;
    const int x_chunks = Mt * (BKS / 8);  // 16-byte chunks of the real X rows of a stage
    // warps that rewrite X rows (whole warps: x_chunks is a multiple of 32)
    const bool x_writer = (dw % GROUP_WARPS) * 32 < x_chunks;

    bool ok = true;
    if constexpr (GIDX) {
      ok = __all_sync(0xffffffffu,
                      mbar_wait_bounded(&bar->tile_full, 0u, abort_flag, kWaitLimitNs));
      if (!ok && lane == 0) record_timeout(err, bar);
    }
    // this thread's column of the scale tile (act order)
    const uint8_t* tile_col = smem + col * 2;
    const uint32_t g_max = (uint32_t)n_groups - 1u;
    // persistent: reads out column block jd (accumulator set jd % 2) and
    // stores its columns of Y; false if the wait expired
    int drained = 0;
    auto drain = [&](int jd) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bar->dblk[jd & 1], (uint32_t)(jd >> 1) & 1u,
                                                     abort_flag, kWaitLimitNs)))
        return false;
      tc_fence_after();
      const int b = (int)blockIdx.x + jd * (int)gridDim.x;
      int l = 0;
      while (l + 1 < ls.count && b >= ls.blk0[l + 1]) ++l;
      const int nl = ls.n[l];
      const int nc = (b - ls.blk0[l]) * BW + col;
      uint16_t* __restrict__ yl = ls.y[l];
      const uint32_t d_set = D_COL + (uint32_t)((jd & 1) * NACC * BT);
      float r[BT];
#pragma unroll
      for (int tb = 0; tb < BT / 16; ++tb) {
        uint32_t v[NACC][16];
#pragma unroll
        for (int c = 0; c < NACC; ++c)
          tmem_ld_32x32b_x16(tmem + lane_addr + d_set + c * BT + 16 * tb, v[c]);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          float acc = __uint_as_float(v[0][q]);
#pragma unroll
          for (int c = 1; c < NACC; ++c) acc += __uint_as_float(v[c][q]);
          r[16 * tb + q] = acc;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->dempty[jd & 1]);  // the set may be overwritten
      if (nc < nl) {
#pragma unroll
        for (int q = 0; q < BT; ++q)
          if (q < Mt) yl[(int64_t)(tok0 + q) * nl + nc] = __half_as_ushort(__float2half_rn(r[q]));
      }
      return true;
    };
    // ring slot and phase of stage t, advanced incrementally (GROUPS <= stages)
    int s = grp % stages;
    uint32_t ph = (uint32_t)(grp / stages) & 1u;
    for (int t = grp; t < n_tot && ok; t += GROUPS, s += GROUPS) {
      if (s >= stages) {
        s -= stages;
        ph ^= 1u;
      }
      if (PERSIST && h == 0) {
        // read out the finished blocks before this stage's block j; those
        // up to j - 2 first of all (block j's MMAs wait for their set)
        const int j = t / n_st;
        while (ok && drained < j) {
          if (drained > j - 2 &&
              !__shfl_sync(0xffffffffu,
                           (int)mbar_test_wait(smem_u32(&bar->dblk[drained & 1]),
                                               (uint32_t)(drained >> 1) & 1u),
                           0))
            break;
          ok = drain(drained);
          ++drained;
        }
        if (!ok) break;
      }
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar->full[s], ph, abort_flag, kWaitLimitNs));
      if (!ok) break;
      uint8_t* st = ring + s * stage_bytes;
      // chunk j: token row j / CPR, 64-k atom (j % CPR) / 8, chunk (j % 8) of
      // the 128-byte row, CPR = BKS / 8 chunks per row (every chunk of the
      // row is permuted, so the swizzle does not matter); rows >= M are zero
      // and stay so
      constexpr int CPR = BKS / 8;
      for (int j = gid; j < x_chunks; j += GROUP_WARPS * 32)
        permute_x_chunk(st + ((j % CPR) >> 3) * X_ATOM_BYTES + (j / CPR) * 128 + (j & 7) * 16);

      if (!PERSIST && t >= n_st) {
        // LoRA stage: one fill.  Row rho (eight ranks) of this slice's chunks
        // comes from lora_b row `col` in the swizzled qweight area and is
        // paired (k, k+4) like X and the dequantised weights.
        const int f = HALVES * n_st + (t - n_st);
        const int a = f % A_SLOTS;
        const uint32_t aph = (uint32_t)(f / A_SLOTS) & 1u;
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
          const int row0 = WPT * (CHUNKS * hs + c);
          const bool mine = row0 < 128 / 8;  // the stage holds 128 ranks: 16 rows
          uint32_t cells[4 * WPT];
          if (mine) {
#pragma unroll
            for (int i = 0; i < WPT; ++i) {
              const int rho = row0 + i;
              const uint4 v = *reinterpret_cast<const uint4*>(
                  st + QW_OFF + (rho >> 3) * LORA_HALF_BYTES + col * 128 +
                  (((rho & 7) ^ (col & 7)) << 4));
              cells[4 * i] = prmt(v.x, v.z, 0x5410);
              cells[4 * i + 1] = prmt(v.x, v.z, 0x7632);
              cells[4 * i + 2] = prmt(v.y, v.w, 0x5410);
              cells[4 * i + 3] = prmt(v.y, v.w, 0x7632);
            }
          }
          if (c == CHUNKS - 1) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->empty[s]);  // lora_b tile of the stage read
          }
          if (c == 0) {
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar->aempty[a], aph ^ 1u, abort_flag,
                                                           kWaitLimitNs));
            if (!ok) break;
            tc_fence_after();
          }
          if (mine)
            tmem_st_32x32b_x32(tmem + lane_addr + A_COL0 + a * A_SLOT_COLS +
                                   4 * WPT * (CHUNKS * hs + c),
                               cells);
        }
        if (!ok) break;
        tmem_wait_st();
        if (x_writer) fence_proxy_async_smem();  // the permuted T rows, for the MMAs
        tc_fence_before();
        mbar_arrive(&bar->afull[a]);
        continue;
      }

#pragma unroll
      for (int hf = 0; hf < HALVES; ++hf) {
        const int f = HALVES * t + hf;  // fill number: A slot f % 3
        const int a = f % A_SLOTS;
        const uint32_t aph = (uint32_t)(f / A_SLOTS) & 1u;
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
          const int row0 = PRA * hf + WPT * (CHUNKS * hs + c);  // first packed row in the stage
          const uint8_t* qw = st + QW_OFF + row0 * (BW * 4) + col * 4;
          const uint8_t* sc = st + S_OFF + col * 2;
          uint32_t cells[4 * WPT];
          uint32_t s2 = 0, zlo = 0, zhi = 0;
          if constexpr (GIDX) {
            // act order: the group of each k from the stage's g_idx slice,
            // its scale from the tile (indices clamped into the tile)
            const uint32_t* gi = reinterpret_cast<const uint32_t*>(st + S_OFF) + 8 * row0;
#pragma unroll
            for (int i = 0; i < WPT; ++i) {
              const uint4 ga = *reinterpret_cast<const uint4*>(gi + 8 * i);
              const uint4 gb = *reinterpret_cast<const uint4*>(gi + 8 * i + 4);
              const uint32_t w = *reinterpret_cast<const uint32_t*>(qw + i * (BW * 4));
              auto sc = [&](uint32_t g) -> uint32_t {
                return *reinterpret_cast<const uint16_t*>(tile_col + min(g, g_max) * S_ROW_BYTES);
              };
              const uint32_t sp[4] = {sc(ga.x) | (sc(gb.x) << 16), sc(ga.y) | (sc(gb.y) << 16),
                                      sc(ga.z) | (sc(gb.z) << 16), sc(ga.w) | (sc(gb.w) << 16)};
              dequant_word_paired_per_pair(w, sp, cells + 4 * i);
            }
          } else if constexpr (!ASYM && WPS >= 4) {
            // symmetric weights, a scale per four or more words: the
            // six-operation form where the scale allows it (same values)
#pragma unroll
            for (int g = 0; g < WPT / WPS; ++g) {
              const int row = (8 * (row0 + WPS * g)) >> gs;
              s2 = half2_broadcast(*reinterpret_cast<const uint16_t*>(sc + row * S_ROW_BYTES));
              uint32_t w[WPS];
#pragma unroll
              for (int i = 0; i < WPS; ++i)
                w[i] = *reinterpret_cast<const uint32_t*>(qw + (WPS * g + i) * (BW * 4));
              if (scale_fits_subnormal_form(s2)) {
                uint32_t b2, c2;
                subnormal_form_constants(s2, b2, c2);
#pragma unroll
                for (int i = 0; i < WPS; ++i)
                  dequant_word_paired_small_scale(w[i], s2, b2, c2, cells + 4 * (WPS * g + i));
              } else {
#pragma unroll
                for (int i = 0; i < WPS; ++i)
                  dequant_word_paired(w[i], s2, cells + 4 * (WPS * g + i));
              }
            }
          } else {
#pragma unroll
          for (int i = 0; i < WPT; ++i) {
            if (i % WPS == 0) {
              // scale row of packed row row0 + i inside the stage's scale tile
              const int row = (8 * (row0 + i)) >> gs;
              s2 = half2_broadcast(*reinterpret_cast<const uint16_t*>(sc + row * S_ROW_BYTES));
              if constexpr (ASYM) {
                const uint32_t zw = *reinterpret_cast<const uint32_t*>(
                    st + z_off + row * Z_ROW_BYTES + (col / 8) * 4);
                const uint32_t z = (zw >> (4 * (col % 8))) & 0xFu;
                zlo = zero_sub_low(z);
                zhi = zero_add_high(z);
              }
            }
            const uint32_t w = *reinterpret_cast<const uint32_t*>(qw + i * (BW * 4));
            uint32_t p[4];
            if constexpr (ASYM)
              dequant_word_paired_z(w, s2, zlo, zhi, p);
            else
              dequant_word_paired(w, s2, p);
#pragma unroll
            for (int j = 0; j < 4; ++j) cells[4 * i + j] = p[j];
          }
          }
          if (hf == HALVES - 1 && c == CHUNKS - 1) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->empty[s]);  // qweight and scales of the stage read
          }
          if (c == 0) {
            // the A slot is free once the MMAs of its previous use have completed
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar->aempty[a], aph ^ 1u, abort_flag,
                                                           kWaitLimitNs));
            if (!ok) break;
            tc_fence_after();
          }
          tmem_st_32x32b_x32(tmem + lane_addr + A_COL0 + a * A_SLOT_COLS +
                                 4 * WPT * (CHUNKS * hs + c),
                             cells);
        }
        if (!ok) break;
        tmem_wait_st();
        if (x_writer && hf == 0) fence_proxy_async_smem();  // the permuted X rows, for the MMAs
        tc_fence_before();
        mbar_arrive(&bar->afull[a]);
      }
    }
    // persistent: the blocks not read out yet
    if (PERSIST && h == 0) {
      while (ok && drained < n_blk) {
        ok = drain(drained);
        ++drained;
      }
    }
    if (!ok && lane == 0) record_timeout(err, bar);

    if (ok) {
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar->dfull, 0, abort_flag, kWaitLimitNs));
      if (!ok && lane == 0) record_timeout(err, bar);
    }
    if (!PERSIST && h == 0) {
      // the four warps of slice 0 hold the four lane quarters: column `col`,
      // tokens in blocks of 16; an empty K range contributes zero
      float* part = reinterpret_cast<float*>(ring);  // [token][column], splits > 1
      if (ok && n_st > 0) tc_fence_after();
#pragma unroll 1
      for (int tb = 0; tb < BT / 16; ++tb) {
        float r[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) r[j] = 0.f;
        if (ok && n_st > 0) {
          // the block's accumulators requested at once, then summed in a fixed order
          uint32_t v[NACC][16];
#pragma unroll
          for (int c = 0; c < NACC; ++c)
            tmem_ld_32x32b_x16(tmem + lane_addr + D_COL + c * BT + 16 * tb, v[c]);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float acc = __uint_as_float(v[0][j]);
#pragma unroll
            for (int c = 1; c < NACC; ++c) acc += __uint_as_float(v[c][j]);
            r[j] = acc;
          }
        }
        if (splits == 1) {
          if (ok && n < N) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (16 * tb + j < Mt)
                y[(int64_t)(tok0 + 16 * tb + j) * N + n] =
                    __half_as_ushort(__float2half_rn(r[j]));
          }
        } else {
          // partial tile in the (fully consumed) ring
#pragma unroll
          for (int j = 0; j < 16; ++j) part[(16 * tb + j) * BW + col] = r[j];
        }
      }
    }
  }

  // Each CTA-wide barrier has a single call site reached by every thread.
  tc_fence_before();
  __syncthreads();
  if (splits > 1) {
    // fixed-order reduction over the cluster's CTAs (consecutive K ranges)
    cluster_sync_all();
    const int rank = (int)cluster_ctarank();
    const int E = Mt * BW;
    const int begin = rank * E / splits, end = (rank + 1) * E / splits;
    const uint32_t base = smem_u32(ring);
    for (int idx = begin + (int)threadIdx.x; idx < end; idx += THREADS) {
      const int tok = idx / BW, c = idx - tok * BW;
      if (n0 + c >= N) continue;
      float sum = 0.f;
      for (int r = 0; r < splits; ++r) sum += ld_dsmem_f32(map_to_rank(base + 4u * idx, r));
      y[(int64_t)(tok0 + tok) * N + n0 + c] = __half_as_ushort(__float2half_rn(sum));
    }
    cluster_sync_all();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int WPS, int BT, int PRS, bool ASYM, bool GIDX, bool PERSIST = false>
cudaError_t launch_t(const CUtensorMap& x_map, const LinearSet& ls, const CUtensorMap& qz_map,
                     const CUtensorMap& t_map, const CUtensorMap& b_map, int lora_rank, int M,
                     int K, int group_shift, int splits, int x3d, const DecodeShape& d,
                     cudaStream_t stream, const DeviceInfo& dev,
                     const LoraFused& lf = LoraFused{}) {
  static std::once_flag once[64];
  static cudaError_t attr_err[64];
  const int di = dev.device & 63;
  std::call_once(once[di], [&] {
    attr_err[di] = cudaFuncSetAttribute(decode_kernel<WPS, BT, PRS, ASYM, GIDX, PERSIST>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        1024 + kRingBudget + 256);
  });
  if (attr_err[di] != cudaSuccess) return attr_err[di];
  cudaLaunchConfig_t cfg = {};
  // persistent: one CTA per SM, each walking several column blocks
  const int blocks = ls.blk0[ls.count];
  const int grid_x = (PERSIST && blocks > dev.num_sms ? dev.num_sms : blocks) + lf.ctas;
  cfg.gridDim = dim3((unsigned)grid_x, (unsigned)splits, (unsigned)d.tok_tiles);
  cfg.blockDim = dim3(THREADS, 1, 1);
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
  return cudaLaunchKernelEx(&cfg, decode_kernel<WPS, BT, PRS, ASYM, GIDX, PERSIST>, x_map, ls,
                            qz_map,
                            t_map, b_map, M, K, group_shift, d.stages, d.stage_bytes,
                            d.scale_rows, x3d, lora_rank, d.n_groups, d.tile_bytes, d.tile_boxes,
                            d.tile_box_rows, lf, dev.error_word);
}

// One linear of a launch, as the host sees it.
struct LinearArgs {
  const int32_t* qweight;
  const uint16_t* scales;
  uint16_t* y;
  int64_t n;
};

// Tensor maps and launch for a token tile of BT over `count` linears that
// share X (count = 1 for a plain call).
// The extras of a single linear: packed zero points for asymmetric weights,
// and a LoRA adapter (t = fp16(x . lora_a^T) [M, rank], lora_b [N, rank]).
struct LinearExtras {
  const int32_t* qzeros = nullptr;
  const uint16_t* t = nullptr;
  const uint16_t* lora_b = nullptr;
  int64_t rank = 0;
  // fused form: T computed in the launch from lora_a; `call` numbers the
  // call on its device (its hand-over slot is call % kTFlagSlots)
  const uint16_t* lora_a = nullptr;
  bool fused = false;
  unsigned long long call = 0;
};

// X as [K/64 atoms][M tokens][64 k] (one box per stage) when K is a multiple
// of 64, else as [M][K] in one box per 64-k atom; rows at or beyond M and k at
// or beyond K read as zero either way.  x3d: which of the two.
template <int BT, int PRS>
bool x_tensor_map(const uint16_t* x, int64_t M, int64_t K, CUtensorMap* x_map, int* x3d) {
  *x3d = 0;
  if (K % 64 == 0) {
    const uint64_t dims[3] = {64, (uint64_t)M, (uint64_t)(K / 64)};
    const uint64_t strides[2] = {(uint64_t)K * 2, 128};
    const uint32_t box[3] = {64, BT, TokGeo<BT, PRS>::X_ATOMS};
    *x3d = tensor_map_3d(x_map, x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B) ? 1 : 0;
  }
  return *x3d || tensor_map_2d(x_map, x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)K,
                               (uint64_t)M, (uint64_t)K * 2, 64, BT, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int BT, int PRS>
cudaError_t launch_bt(const uint16_t* x, const LinearArgs* lin, int count,
                      const LinearExtras& ex, int64_t M, int64_t K, int group_shift, int splits,
                      cudaStream_t stream, const DeviceInfo& dev) {
  const int32_t* qzeros = ex.qzeros;
  const bool asym = qzeros != nullptr;
  if ((asym || ex.rank > 0) && count != 1) return cudaErrorInvalidValue;
  if (ex.rank > 0 && !TokGeo<BT, PRS>::LORA_OK) return cudaErrorInvalidValue;
  const DecodeShape d = decode_shape<BT, PRS>(group_shift, asym);
  if (d.stages < GROUPS || d.smem_bytes > 1024 + kRingBudget + 256) return cudaErrorInvalidValue;
  if (count < 1 || count > kMaxLinears) return cudaErrorInvalidValue;
  const int64_t n_groups = (group_shift == 62 || (int64_t(1) << group_shift) >= K)
                               ? 1 : (K + (int64_t(1) << group_shift) - 1) >> group_shift;
  LinearSet ls;
  ls.count = count;
  ls.blk0[0] = 0;
  for (int i = 0; i < count; ++i) {
    const uint64_t N = (uint64_t)lin[i].n;
    if (!tensor_map_2d(&ls.qw[i], lin[i].qweight, CU_TENSOR_MAP_DATA_TYPE_INT32, N,
                       (uint64_t)(K / 8), N * 4, BW, PRS, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !tensor_map_2d(&ls.sc[i], lin[i].scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, N,
                       (uint64_t)n_groups, N * 2, BW, (uint32_t)d.scale_rows,
                       CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    ls.y[i] = lin[i].y;
    ls.n[i] = (int)N;
    ls.blk0[i + 1] = ls.blk0[i] + (int)((N + BW - 1) / BW);
  }
  for (int i = count; i < kMaxLinears; ++i) {
    ls.qw[i] = ls.qw[0];
    ls.sc[i] = ls.sc[0];
    ls.y[i] = nullptr;
    ls.n[i] = 0;
    ls.blk0[i + 1] = ls.blk0[count];
  }
  CUtensorMap x_map;
  int x3d = 0;
  if (!x_tensor_map<BT, PRS>(x, M, K, &x_map, &x3d)) return cudaErrorInvalidValue;
  CUtensorMap qz_map = ls.qw[0];  // read only for asymmetric weights
  if (asym) {
    const uint64_t N = (uint64_t)lin[0].n;
    if (!tensor_map_2d(&qz_map, qzeros, CU_TENSOR_MAP_DATA_TYPE_INT32, N / 8, (uint64_t)n_groups,
                       N / 2, BW / 8, (uint32_t)d.scale_rows, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  // LoRA: T [M, rank] as 64-rank atoms of BT rows (the X layout), lora_b
  // [N, rank] as 64-rank halves of 128 rows; both with the 128-byte swizzle
  CUtensorMap t_map = x_map, b_map = x_map;  // read only with an adapter
  const int lora_rank = (int)ex.rank;
  if (lora_rank > 0) {
    const uint64_t N = (uint64_t)lin[0].n;
    if (!tensor_map_2d(&t_map, ex.t, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)lora_rank,
                       (uint64_t)M, (uint64_t)lora_rank * 2, 64, BT, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tensor_map_2d(&b_map, ex.lora_b, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)lora_rank, N,
                       (uint64_t)lora_rank * 2, 64, BW, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  if (splits <= 0) splits = decode_pick_splits_blocks(ls.blk0[count], K, PRS, dev);
  // with an adapter, the last split's CTA (which runs the LoRA stages after
  // its K stages) must own at least one K stage: the first MMAs of its K
  // stages are what initialise its accumulators
  if (lora_rank > 0) {
    const int ns = (int)(((K >> 3) + PRS - 1) / PRS);
    if (splits > ns) splits = ns;
  }
  // fused form: T CTAs on the SMs the column blocks leave free (each CTA of
  // the layer's grid takes an SM), at most one per rank
  LoraFused lf{};
  if (ex.fused) {
    const int ctas = std::min<int>((dev.num_sms - ls.blk0[count] * splits) / splits, lora_rank);
    if (ctas < 1 || !ex.lora_a) return cudaErrorInvalidValue;
    // the CTAs with adapter stages: the last split of every column block
    lf = LoraFused{x, ex.lora_a, const_cast<uint16_t*>(ex.t), dev.t_flags + ex.call % kTFlagSlots,
                   ctas, ls.blk0[count], lora_rank};
  }
  const int iM = (int)M, iK = (int)K;
  const int gsh = group_shift;
  if (asym) {
    if (gsh == 4)
      return launch_t<2, BT, PRS, true, false>(x_map, ls, qz_map, t_map, b_map, lora_rank, iM,
                                               iK, gsh, splits, x3d, d, stream, dev);
    if (gsh == 5)
      return launch_t<4, BT, PRS, true, false>(x_map, ls, qz_map, t_map, b_map, lora_rank, iM,
                                               iK, gsh, splits, x3d, d, stream, dev);
    return launch_t<WPT, BT, PRS, true, false>(x_map, ls, qz_map, t_map, b_map, lora_rank, iM,
                                               iK, gsh, splits, x3d, d, stream, dev);
  }
  // more column blocks than SMs (wide or grouped linears) at up to 16 tokens
  // without a split: one persistent wave instead of several
  if constexpr (BT == 16 && PRS == 2 * PRA) {
    if (splits == 1 && lora_rank == 0 && ls.blk0[count] > dev.num_sms) {
      if (gsh == 4)
        return launch_t<2, BT, PRS, false, false, true>(x_map, ls, qz_map, t_map, b_map, 0, iM,
                                                        iK, gsh, splits, x3d, d, stream, dev);
      if (gsh == 5)
        return launch_t<4, BT, PRS, false, false, true>(x_map, ls, qz_map, t_map, b_map, 0, iM,
                                                        iK, gsh, splits, x3d, d, stream, dev);
      return launch_t<WPT, BT, PRS, false, false, true>(x_map, ls, qz_map, t_map, b_map, 0, iM,
                                                        iK, gsh, splits, x3d, d, stream, dev);
    }
  }
  if (gsh == 4)
    return launch_t<2, BT, PRS, false, false>(x_map, ls, qz_map, t_map, b_map, lora_rank, iM, iK,
                                              gsh, splits, x3d, d, stream, dev, lf);
  if (gsh == 5)
    return launch_t<4, BT, PRS, false, false>(x_map, ls, qz_map, t_map, b_map, lora_rank, iM, iK,
                                              gsh, splits, x3d, d, stream, dev, lf);
  return launch_t<WPT, BT, PRS, false, false>(x_map, ls, qz_map, t_map, b_map, lora_rank, iM, iK,
                                              gsh, splits, x3d, d, stream, dev, lf);
}

cudaError_t launch_set(const uint16_t* x, const LinearArgs* lin, int count,
                       const LinearExtras& ex, int64_t M, int64_t K, int group_shift, int splits,
                       cudaStream_t stream, const DeviceInfo& dev) {
  int64_t nblk = 0;
  for (int i = 0; i < count; ++i) nblk += (lin[i].n + BW - 1) / BW;
  const bool wide = decode_stage_rows(M, nblk, K, splits, ex.rank > 0, dev) == 2 * PRA;
  // token tile: the smallest of 16, 32, 48 and 64 that holds M
  if (M <= 16)
    return wide ? launch_bt<16, 2 * PRA>(x, lin, count, ex, M, K, group_shift, splits, stream, dev)
                : launch_bt<16, PRA>(x, lin, count, ex, M, K, group_shift, splits, stream, dev);
  if (M <= 32)
    return wide ? launch_bt<32, 2 * PRA>(x, lin, count, ex, M, K, group_shift, splits, stream, dev)
                : launch_bt<32, PRA>(x, lin, count, ex, M, K, group_shift, splits, stream, dev);
  if (ex.rank > 0) return cudaErrorInvalidValue;  // adapters: up to 32 tokens
  if (M <= 48) return launch_bt<48, PRA>(x, lin, count, ex, M, K, group_shift, splits, stream, dev);
  return launch_bt<64, PRA>(x, lin, count, ex, M, K, group_shift, splits, stream, dev);
}

// Act order on a token tile of BT: false if the scale tile leaves no room
// for two ring stages.
template <int BT, int PRS>
bool gidx_fits(int64_t n_groups) {
  return decode_shape_gidx<BT, PRS>(n_groups).stages >= GROUPS;
}

template <int BT, int PRS>
cudaError_t launch_gidx_bt(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                           const int32_t* g_idx, uint16_t* y, int64_t M, int64_t K, int64_t N,
                           int64_t n_groups, cudaStream_t stream, const DeviceInfo& dev) {
  DecodeShape d = decode_shape_gidx<BT, PRS>(n_groups);
  if (d.stages < GROUPS) return cudaErrorInvalidValue;
  d.tok_tiles = (int)((M + BT - 1) / BT);
  LinearSet ls;
  ls.count = 1;
  ls.blk0[0] = 0;
  if (!tensor_map_2d(&ls.qw[0], qweight, CU_TENSOR_MAP_DATA_TYPE_INT32, (uint64_t)N,
                     (uint64_t)(K / 8), (uint64_t)N * 4, BW, PRS, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !tensor_map_2d(&ls.sc[0], scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, (uint64_t)N,
                     (uint64_t)n_groups, (uint64_t)N * 2, BW, (uint32_t)d.tile_box_rows,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  ls.y[0] = y;
  ls.n[0] = (int)N;
  ls.blk0[1] = (int)((N + BW - 1) / BW);
  for (int i = 1; i < kMaxLinears; ++i) {
    ls.qw[i] = ls.qw[0];
    ls.sc[i] = ls.sc[0];
    ls.y[i] = nullptr;
    ls.n[i] = 0;
    ls.blk0[i + 1] = ls.blk0[1];
  }
  CUtensorMap x_map, gi_map;
  int x3d = 0;
  if (!x_tensor_map<BT, PRS>(x, M, K, &x_map, &x3d)) return cudaErrorInvalidValue;
  // g_idx [K] as [K / 16 rows x 16]: one box of a stage's BKS entries
  if (!tensor_map_2d(&gi_map, g_idx, CU_TENSOR_MAP_DATA_TYPE_INT32, 16, (uint64_t)(K / 16), 64,
                     16, TokGeo<BT, PRS>::BKS / 16, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const int splits = decode_pick_splits_blocks((int64_t)ls.blk0[1] * d.tok_tiles, K, PRS, dev);
  return launch_t<WPT, BT, PRS, false, true>(x_map, ls, gi_map, x_map, x_map, 0, (int)M, (int)K,
                                             62, splits, x3d, d, stream, dev);
}

}  // namespace

int decode_pick_splits_blocks(int64_t nblk, int64_t K, int prs, const DeviceInfo& dev) {
  // One CTA per SM.  Pick the split that minimises (waves of CTAs) x (stages
  // per CTA) plus one stage for the cluster reduction, among splits whose
  // CTAs are all resident at once.  Ties go to the smaller split.
  const int64_t ns = ((K >> 3) + prs - 1) / prs;
  const int64_t sms = dev.num_sms;
  int best = 1;
  int64_t best_cost = -1;
  for (int s = 1; s <= 8; ++s) {
    if (s > 1 && (nblk * s > sms || ns < s)) break;
    const int64_t waves = (nblk * s + sms - 1) / sms;
    const int64_t cost = waves * ((ns + s - 1) / s) + (s > 1 ? 1 : 0);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

int decode_stage_rows(int64_t M, int64_t nblk, int64_t K, int splits, bool lora,
                      const DeviceInfo& dev) {
  // An adapter's stages need the 512-k stage's qweight area (two 64-rank
  // lora_b halves).  Otherwise the 16-token tile streams 512-k stages (four
  // fit the ring) when each CTA takes the whole K range of its columns, where
  // fewer, larger copies cost less per byte, and 256-k stages (eight) when the
  // K range is split, where a CTA's share is short and the ring's fill and
  // drain weigh more.  Larger tiles take 256-k stages: their X tiles leave
  // room for only two or three 512-k stages.
  if (lora) return 2 * PRA;
  if (M > 16) return PRA;
  const int s = splits > 0 ? splits : decode_pick_splits_blocks(nblk, K, 2 * PRA, dev);
  return s == 1 ? 2 * PRA : PRA;
}

int decode_pick_splits(int64_t M, int64_t K, int64_t N, bool lora, const DeviceInfo& dev) {
  const int64_t nblk = (N + BW - 1) / BW;
  return decode_pick_splits_blocks(nblk, K, decode_stage_rows(M, nblk, K, 0, lora, dev), dev);
}

int64_t decode_ctas(int64_t M, int64_t K, int64_t N, bool lora, const DeviceInfo& dev) {
  return (N + BW - 1) / BW * decode_pick_splits(M, K, N, lora, dev);
}

cudaError_t launch_decode(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                          uint16_t* y, int64_t M, int64_t K, int64_t N, int group_shift,
                          int splits, cudaStream_t stream, const DeviceInfo& dev) {
  const LinearArgs one{qweight, scales, y, N};
  return launch_set(x, &one, 1, LinearExtras{}, M, K, group_shift, splits, stream, dev);
}

cudaError_t launch_decode_asym(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                               const int32_t* qzeros, uint16_t* y, int64_t M, int64_t K,
                               int64_t N, int group_shift, cudaStream_t stream,
                               const DeviceInfo& dev) {
  const LinearArgs one{qweight, scales, y, N};
  LinearExtras ex;
  ex.qzeros = qzeros;
  return launch_set(x, &one, 1, ex, M, K, group_shift, 0, stream, dev);
}

cudaError_t launch_decode_lora(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                               uint16_t* y, int64_t M, int64_t K, int64_t N, int group_shift,
                               const uint16_t* t, const uint16_t* lora_b, int64_t rank,
                               cudaStream_t stream, const DeviceInfo& dev) {
  const LinearArgs one{qweight, scales, y, N};
  LinearExtras ex;
  ex.t = t;
  ex.lora_b = lora_b;
  ex.rank = rank;
  return launch_set(x, &one, 1, ex, M, K, group_shift, 0, stream, dev);
}

cudaError_t launch_decode_gidx(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                               const int32_t* g_idx, uint16_t* y, int64_t M, int64_t K,
                               int64_t N, int64_t n_groups, cudaStream_t stream,
                               const DeviceInfo& dev) {
  // Token tile as for plain weights (64 at most; more tokens take several
  // tiles along the grid's z), and the stage size of the plain layer where
  // the scale tile leaves room for it, so that consecutive group indices give
  // the plain layer's result bit for bit.  Otherwise 256-k stages, else a
  // smaller token tile.
  const int64_t nblk = (N + BW - 1) / BW;
  const int64_t mt = M < 64 ? M : 64;
  const bool wide = decode_stage_rows(mt, nblk, K, 0, false, dev) == 2 * PRA;
  const auto args = [&](auto launch) {
    return launch(x, qweight, scales, g_idx, y, M, K, N, n_groups, stream, dev);
  };
  if (mt <= 16 && wide && gidx_fits<16, 2 * PRA>(n_groups))
    return args(launch_gidx_bt<16, 2 * PRA>);
  if (mt > 48 && gidx_fits<64, PRA>(n_groups)) return args(launch_gidx_bt<64, PRA>);
  if (mt > 32 && gidx_fits<48, PRA>(n_groups)) return args(launch_gidx_bt<48, PRA>);
  if (mt > 16 && gidx_fits<32, PRA>(n_groups)) return args(launch_gidx_bt<32, PRA>);
  if (gidx_fits<16, PRA>(n_groups)) return args(launch_gidx_bt<16, PRA>);
  return cudaErrorInvalidValue;
}

bool decode_lora_fused_fits(int64_t M, int64_t K, int64_t N, int64_t rank,
                            const DeviceInfo& dev) {
  if (M < 1 || M > 32 || rank < 1) return false;
  // the adapter's launch geometry: 512-k stages, the split decode_pick_splits
  // gives them, at most one per K stage
  const int64_t nblk = (N + BW - 1) / BW;
  int splits = decode_pick_splits_blocks(nblk, K, 2 * PRA, dev);
  const int ns = (int)(((K >> 3) + 2 * PRA - 1) / (2 * PRA));
  if (splits > ns) splits = ns;
  const int64_t ctas = std::min<int64_t>((dev.num_sms - nblk * splits) / splits, rank);
  if (ctas < 1) return false;
  // A T CTA's time is a chain of load latencies: its busiest warp takes
  // ceil(ranks per CTA x 256-k pieces / warps) pieces, each in rounds of
  // eight tokens.  Measured on the up-projection: up to 16 rounds the T CTAs
  // finish under the layer's K stages (rank 32 at 1 to 32 tokens, rank 128
  // at up to 8); beyond that the separate T launch is faster.
  constexpr int64_t kWarps = THREADS / 32;
  const int64_t ranks = (rank + ctas - 1) / ctas;
  const int64_t pieces = (K + 255) / 256;
  const int64_t rounds = (ranks * pieces + kWarps - 1) / kWarps * ((M + 7) / 8);
  return rounds <= 16;
}

cudaError_t launch_decode_lora_fused(const uint16_t* x, const int32_t* qweight,
                                     const uint16_t* scales, uint16_t* y, int64_t M, int64_t K,
                                     int64_t N, int group_shift, uint16_t* t,
                                     const uint16_t* lora_a, const uint16_t* lora_b,
                                     int64_t rank, cudaStream_t stream, const DeviceInfo& dev) {
  static std::atomic<unsigned long long> calls[64];
  const LinearArgs one{qweight, scales, y, N};
  LinearExtras ex;
  ex.t = t;
  ex.lora_b = lora_b;
  ex.rank = rank;
  ex.lora_a = lora_a;
  ex.fused = true;
  ex.call = ++calls[dev.device & 63];
  return launch_set(x, &one, 1, ex, M, K, group_shift, 0, stream, dev);
}

cudaError_t launch_decode_grouped(const uint16_t* x, const int32_t* const* qweights,
                                  const uint16_t* const* scales, const int64_t* ns,
                                  uint16_t* const* ys, int count, int64_t M, int64_t K,
                                  int group_shift, cudaStream_t stream, const DeviceInfo& dev) {
  if (count < 1 || count > kMaxLinears) return cudaErrorInvalidValue;
  LinearArgs lin[kMaxLinears];
  for (int i = 0; i < count; ++i) lin[i] = LinearArgs{qweights[i], scales[i], ys[i], ns[i]};
  return launch_set(x, lin, count, LinearExtras{}, M, K, group_shift, 0, stream, dev);
}

}  // namespace gptq
