// Prefill kernel on CTA pairs: Y[M, N] = X[M, K] . dequant(qweight, scales)
// with tcgen05.mma.cta_group::2, for token tiles of 128 or 256.
//
// Operation: GPTQ-Pro README, "Runtime contract" and "Ampere kernel
// architecture" (tensor-core prefill with FP32 accumulation that reads the
// native int32 qweight; predicated tails; FP16 output).  The Ampere design is
// prior art only.
//
// Same transposed product as the single-CTA prefill kernel (Y^T = W^T . X^T:
// weights are the MMA's A operand from TMEM, tokens its N dimension), but the
// two CTAs of a cluster share one 256-column x BT-token tile:
//
// * each CTA dequantises its own 128 weight columns into its own TMEM (A rows
//   0..127 live in the even CTA, rows 128..255 in the odd one);
// * each CTA loads only HALF of the X tile (BT/2 token rows x 128 k per
//   stage); the pair MMA reads B rows 0..BT/2-1 from the even CTA and the
//   rest from the odd CTA, so every X byte crosses from L2 once per pair
//   instead of once per CTA;
// * one thread of the even CTA issues the M = 256 MMAs; their completion is
//   signalled to the barriers of both CTAs at once (tcgen05.commit with a
//   CTA mask).  Both CTAs' X loads count their bytes on the even CTA's
//   barrier, and both CTAs' dequantisation warps arrive on the even CTA's
//   A-slot barrier.
//
// Halving the X traffic per SM matters because moving X from L2 into shared
// memory is where most of the power of this kernel goes: with half of it the
// SMs hold a higher clock under the board's power limit.
//
// The kernel is persistent: one cluster per SM pair walks the tiles (column
// pair fastest), and every ring continues across tiles.  The accumulator is
// drained by the dequantisation warps between two of their stages: each
// group reads its quarter of the tokens from TMEM, hands the accumulator back
// to the MMA warp at once, then rounds to FP16 into a shared-memory staging
// tile that one TMA store writes to Y.  So the next tile's copies,
// dequantisation and MMAs overlap the previous tile's epilogue, and no CTA
// launch, TMEM allocation or pipeline fill is paid per tile.
//
// With asymmetric zero points (ASYM; GPTQModel wiki, "Defaults and
// compatibility decisions": sym) the weight producer also loads the stage's
// rows of packed zeros (qzeros [n_groups, N/8], eight per int32 along N) and
// the dequantisation subtracts each column's zero instead of 8, at the same
// number of FP16 operations.
//
// With a LoRA adapter (GPTQ-Pro README, "Runtime contract": adapters on the
// linear path) each tile gets rank/32 more stages after its K stages: the
// weight producer loads 32 columns of lora_b (FP16, copied into the TMEM A
// slot as they are), the X producer loads the same 32 columns of T =
// fp16(X . lora_a^T), and the MMAs add T . lora_b^T into the same FP32
// accumulator, so Y is rounded once.
//
// Every wait is bounded in time; on expiry the CTA records GPTQ_ERR_TIMEOUT
// in the device error word and winds down.  Both CTAs always reach the final
// cluster barrier, so neither leaves while the other may still signal it.

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc05.cuh"
#include "tmap.h"

namespace gptq {

namespace {

constexpr int BW = 128;   // weight columns per CTA (TMEM lanes); 256 per pair (MMA M)
constexpr int BK = 128;   // k per pipeline stage (eight k16 MMAs)
constexpr int XS_MAX = 4;   // X ring stages (half tile per CTA), at most
constexpr int WS_MAX = 12;  // weight-tile ring stages (qweight + scales of 128 k), at most
constexpr int AS = 4;       // A slots in TMEM (128 k each)
constexpr int DQ_GROUPS = 4;             // dequantisation groups: group g takes stages g mod 4
constexpr int DQ_WARPS = 4 * DQ_GROUPS;  // one warp per TMEM lane quarter in each group
constexpr int DQ_WARP0 = 3;  // warps 0, 1, 2: X producer, MMA issuer, weight producer
constexpr int THREADS = (DQ_WARP0 + DQ_WARPS) * 32;
constexpr int QW_STAGE_BYTES = BW * (BK / 8) * 4;  // 128 columns x 16 packed rows: 8 KB
constexpr int S_ROW_BYTES = BW * 2;                // one scale row of the tile: 256 B
constexpr int S_STAGE_MAX_ROWS = BK / 16;          // group 16: eight rows per stage
constexpr int Z_ROW_BYTES = BW / 8 * 4;           // one row of packed zero points: 64 B
constexpr int Z_OFF = QW_STAGE_BYTES + S_STAGE_MAX_ROWS * S_ROW_BYTES;  // zeros in a slot
constexpr int W_STAGE_BYTES = Z_OFF + S_STAGE_MAX_ROWS * Z_ROW_BYTES;
// A LoRA stage: 32 of the adapter's rank.  Its weight tile is lora_b's 128
// rows x 32 FP16 (64-byte rows, no swizzle); its token tile is T's rows x 64
// columns (128-byte swizzle; the 32 columns past the stage are not used).
constexpr int LORA_R = 32;
constexpr int LORA_W_BYTES = BW * LORA_R * 2;
static_assert(LORA_W_BYTES <= W_STAGE_BYTES, "a LoRA weight tile fits a weight slot");
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t D_COL = 0;              // accumulator: columns [0, BT)
constexpr uint32_t A_COL = 256;            // A slots: [256, 256 + 4 * 64)
constexpr uint32_t A_STAGE_COLS = BK / 2;  // two FP16 per 32-bit column
constexpr uint16_t kPairMask = 0x3;        // both CTAs of the cluster
constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr uint64_t kDrainLimitNs = 200000000ull;
static_assert(A_COL + AS * A_STAGE_COLS <= TMEM_COLS, "TMEM budget");
static_assert(AS == DQ_GROUPS, "stage g uses A slot g mod 4 and is dequantised by group g mod 4");

// Ring depths and shared-memory layout for a pair token tile of BT (BT/2 X
// rows per CTA).  The weight ring is as deep as shared memory allows: below
// a few token tiles every weight stage comes from HBM, and the bytes a CTA
// keeps in flight set its streaming rate.
// An X stage is two 64-k halves, each BT/2 rows of 128 bytes (128-byte
// swizzle), the second right after the first.  The staging area holds this
// CTA's 128 columns x BT tokens of Y in FP16: one block of BT/4 tokens x 32
// columns (token-major, 64-byte rows) per dequantisation warp, which stores
// it to Y on its own.
template <int BT>
struct PairLayout {
  static constexpr int XS = BT == 256 ? 3 : 4;
  static constexpr int WS = BT == 256 ? 4 : 8;
  static constexpr int HT = BT / 2;
  static constexpr int TPG = BT / DQ_GROUPS;  // tokens drained per group
  static constexpr int X_HALF_BYTES = HT * 64 * 2;
  static constexpr int X_STAGE_BYTES = 2 * X_HALF_BYTES;
  static constexpr int W_OFF = XS * X_STAGE_BYTES;
  static constexpr int Y_OFF = W_OFF + WS * W_STAGE_BYTES;
  static constexpr int Y_WARP_BYTES = TPG * 32 * 2;
  static constexpr int Y_GROUP_BYTES = 4 * Y_WARP_BYTES;
  static constexpr int BAR_OFF = Y_OFF + DQ_GROUPS * Y_GROUP_BYTES;
  static constexpr size_t kSmemBytes = 1024 + (size_t)BAR_OFF + 512;
  static_assert(X_HALF_BYTES % 1024 == 0, "128-byte swizzle atoms stay aligned");
  static_assert(Y_OFF % 128 == 0 && Y_WARP_BYTES % 128 == 0, "store sources aligned");
  static_assert(TPG % 32 == 0, "drained in 32-column TMEM loads");
  static_assert(XS <= XS_MAX && WS <= WS_MAX && WS % DQ_GROUPS == 0,
                "weight slot g mod WS is always used by group g mod 4");
};

// Both CTAs hold the full set; xfull, afull and dempty are only used in the
// even CTA.
struct PairBarriers {
  uint64_t xfull[XS_MAX];   // both halves of the X stage landed (even CTA)
  uint64_t xempty[XS_MAX];  // pair MMAs reading the X stage done
  uint64_t wfull[WS_MAX];   // this CTA's qweight and scale tiles landed
  uint64_t wempty[WS_MAX];  // weight tiles read by this CTA's group warps
  uint64_t afull[AS];   // A slot written by the group warps of both CTAs (even CTA)
  uint64_t aempty[AS];  // pair MMAs reading the A slot done
  uint64_t dfull;       // all MMAs of the current tile done
  uint64_t dempty;      // accumulator read out by every group warp of both CTAs (even CTA)
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(PairBarriers) <= 512, "barrier area");

// The tiles of one cluster: tile = cluster + i * clusters for i = 0, 1, ...;
// column pair fastest.
struct TileWalk {
  int cluster, clusters, n_pairs, tiles;
  __device__ int count() const {
    return cluster < tiles ? (tiles - cluster + clusters - 1) / clusters : 0;
  }
  __device__ void coords(int i, int bt, uint32_t rank, int& n0, int& t0) const {
    const int tile = cluster + i * clusters;
    n0 = (2 * (tile % n_pairs) + (int)rank) * BW;
    t0 = (tile / n_pairs) * bt;
  }
};

// scale_rows: scale rows one 128-k stage touches (1, or 128/group for groups
// below 128); stages start on 128-k boundaries, so they align with groups.
// x3d: X is read through a [K/64][M][64] view, one copy per stage (K a
// multiple of 64); otherwise through [M][K], one copy per 64-k half.
// n_pairs, tiles: column pairs (of 256) and pair tiles (n_pairs x token
// tiles); cluster c takes tiles c, c + clusters, ...
// lora_stages: LoRA stages per tile (0 without an adapter); t_map and b_map
// then describe T [M, rank] and lora_b [N, rank].
template <int BT, bool ASYM>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    prefill_pair_kernel(const __grid_constant__ CUtensorMap x_map,
                        const __grid_constant__ CUtensorMap qw_map,
                        const __grid_constant__ CUtensorMap s_map,
                        const __grid_constant__ CUtensorMap qz_map,
                        const __grid_constant__ CUtensorMap y_map,
                        const __grid_constant__ CUtensorMap t_map,
                        const __grid_constant__ CUtensorMap b_map, int M, int K, int N,
                        int group_shift, int scale_rows, int x3d, int n_pairs, int tiles,
                        int lora_stages, int* err) {
  static_assert(BT == 128 || BT == 256, "pair token tile");
  using L = PairLayout<BT>;
  constexpr int HT = L::HT;
  constexpr int TPG = L::TPG;
  constexpr int XS = L::XS;
  constexpr int WS = L::WS;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base; the same offset in both CTAs, so that one MMA
  // descriptor and one barrier offset name the matching buffers of the pair
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* xs = smem;
  PairBarriers* bar = reinterpret_cast<PairBarriers*>(smem + L::BAR_OFF);
  volatile int* abort_flag = &bar->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: even CTA (issues the MMAs), 1: odd CTA
  const bool even = rank == 0;
  const TileWalk walk{(int)(blockIdx.x >> 1), (int)(gridDim.x >> 1), n_pairs, tiles};
  const int NT = walk.count();          // tiles of this cluster
  const int KW = (K + BK - 1) / BK;     // weight stages per tile
  const int KB = KW + lora_stages;      // stages per tile (weights, then LoRA)
  const int G = NT * KB;                // stages of this cluster, over all its tiles

  if (threadIdx.x == 0) {
    for (int s = 0; s < XS; ++s) {
      mbar_init(&bar->xfull[s], 1);   // the even CTA's expect_tx; bytes from both CTAs
      mbar_init(&bar->xempty[s], 1);  // one pair commit
    }
    for (int j = 0; j < WS; ++j) {
      mbar_init(&bar->wfull[j], 1);
      mbar_init(&bar->wempty[j], 4);      // the four warps of the slot's group
    }
    for (int j = 0; j < AS; ++j) {
      mbar_init(&bar->afull[j], 2 * 4);   // the slot's group warps in both CTAs
      mbar_init(&bar->aempty[j], 1);      // one pair commit
    }
    mbar_init(&bar->dfull, 1);                 // one pair commit per tile
    mbar_init(&bar->dempty, 2 * DQ_WARPS);     // every group warp of both CTAs
    bar->abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&x_map);
    prefetch_tensormap(&qw_map);
    prefetch_tensormap(&s_map);
    prefetch_tensormap(&y_map);
    if (ASYM) prefetch_tensormap(&qz_map);
    if (lora_stages > 0) {
      prefetch_tensormap(&t_map);
      prefetch_tensormap(&b_map);
    }
  }
  __syncwarp();
  if (warp == 1) {
    tmem_alloc_pair(&bar->tmem_base, TMEM_COLS);
    tmem_relinquish_pair();
  }
  // both CTAs' barriers are initialised and TMEM is allocated before any
  // thread signals the other CTA
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  // the even CTA's barriers that both CTAs signal
  const uint32_t xfull_even = map_to_rank(smem_u32(&bar->xfull[0]), 0);
  const uint32_t afull_even = map_to_rank(smem_u32(&bar->afull[0]), 0);
  const uint32_t dempty_even = map_to_rank(smem_u32(&bar->dempty), 0);

  if (warp == 0 || warp == 2) {
    // ---------------- TMA producers: X half (warp 0), weights (warp 2) ----------------
    // One thread each.  The loops are kept lean (ring depth known at compile
    // time, slot and phase advanced incrementally, per-tile values hoisted):
    // below a few hundred tokens the MMAs are short and the issue rate of
    // these threads sets the pace.
    if (lane == 0 && NT > 0) {
      int it = 0, kb = 0, n0, t0;
      walk.coords(0, BT, rank, n0, t0);
      int s = 0;
      uint32_t ph = 0;
      int issued = 0;
      if (warp == 0) {
        // Does the odd CTA's half of the token tile hold any row below M?
        // If not, it loads nothing (no copy box lies wholly outside X) and
        // the even CTA expects only its own bytes; the MMA then reads stale
        // shared memory for token columns that are never stored.
        bool odd_rows = t0 + HT < M;
        bool load = even || odd_rows;
        uint32_t copies = odd_rows ? 2u : 1u;
        int row = t0 + (int)rank * HT;
        bool t_ready = false;
        for (int g = 0; g < G; ++g) {
          if (!mbar_wait_bounded(&bar->xempty[s], ph ^ 1u, abort_flag, kWaitLimitNs)) {
            record_timeout(err, bar);
            break;
          }
          uint8_t* dst = xs + s * L::X_STAGE_BYTES;
          const uint32_t bar_c = xfull_even + 8u * (uint32_t)s;
          if (kb < KW) {
            const int k0 = kb * BK;
            // the second 64-k half holds k below K (else it is neither loaded
            // nor multiplied)
            const bool hi = k0 + 64 < K;
            if (even)
              mbar_arrive_expect_tx(&bar->xfull[s],
                                    copies * ((x3d || hi) ? L::X_STAGE_BYTES : L::X_HALF_BYTES));
            if (load) {
              if (x3d) {
                tma_load_3d_pair(dst, &x_map, 0, row, k0 / 64, bar_c);
              } else {
                tma_load_2d_pair(dst, &x_map, k0, row, bar_c);
                if (hi) tma_load_2d_pair(dst + L::X_HALF_BYTES, &x_map, k0 + 64, row, bar_c);
              }
            }
          } else {
            // LoRA stage: 64 columns of T from column 32 * (kb - KW).  T comes
            // from the launch before this one, which may still be running
            // (programmatic dependent launch): wait for it once, here.
            if (!t_ready) {
              asm volatile("griddepcontrol.wait;" ::: "memory");
              t_ready = true;
            }
            if (even) mbar_arrive_expect_tx(&bar->xfull[s], copies * L::X_HALF_BYTES);
            if (load) tma_load_2d_pair(dst, &t_map, LORA_R * (kb - KW), row, bar_c);
          }
          ++issued;
          if (++s == XS) {
            s = 0;
            ph ^= 1u;
          }
          if (++kb == KB) {
            kb = 0;
            if (++it < NT) {
              walk.coords(it, BT, rank, n0, t0);
              odd_rows = t0 + HT < M;
              load = even || odd_rows;
              copies = odd_rows ? 2u : 1u;
              row = t0 + (int)rank * HT;
            }
          }
        }
        if (*abort_flag && even) {
          // drain: wait for the last loads issued into each slot (the odd
          // CTA's X loads complete on the even CTA's barriers, which the
          // even CTA drains)
          int never = 0;
          for (int j = issued - 1; j >= 0 && j >= issued - XS; --j)
            mbar_wait_bounded(&bar->xfull[j % XS], (uint32_t)(j / XS) & 1u, &never,
                              kDrainLimitNs);
        }
      } else {
        const uint32_t wbytes =
            QW_STAGE_BYTES + scale_rows * (S_ROW_BYTES + (ASYM ? Z_ROW_BYTES : 0));
        uint8_t* wst = smem + L::W_OFF;
        for (int g = 0; g < G; ++g) {
          if (!mbar_wait_bounded(&bar->wempty[s], ph ^ 1u, abort_flag, kWaitLimitNs)) {
            record_timeout(err, bar);
            break;
          }
          if (n0 < N && kb < KW) {
            const int k0 = kb * BK;
            mbar_arrive_expect_tx(&bar->wfull[s], wbytes);
            tma_load_2d(wst, &qw_map, n0, k0 / 8, &bar->wfull[s]);
            tma_load_2d(wst + QW_STAGE_BYTES, &s_map, n0, (int)((int64_t)k0 >> group_shift),
                        &bar->wfull[s]);
            if (ASYM)
              tma_load_2d(wst + Z_OFF, &qz_map, n0 / 8, (int)((int64_t)k0 >> group_shift),
                          &bar->wfull[s]);
          } else if (n0 < N) {
            // LoRA stage: lora_b rows n0.. , columns 32 * (kb - KW) ..
            mbar_arrive_expect_tx(&bar->wfull[s], LORA_W_BYTES);
            tma_load_2d(wst, &b_map, LORA_R * (kb - KW), n0, &bar->wfull[s]);
          } else {
            mbar_arrive(&bar->wfull[s]);  // padding CTA: no columns, nothing to load
          }
          ++issued;
          wst += W_STAGE_BYTES;
          if (++s == WS) {
            s = 0;
            ph ^= 1u;
            wst = smem + L::W_OFF;
          }
          if (++kb == KB) {
            kb = 0;
            if (++it < NT) walk.coords(it, BT, rank, n0, t0);
          }
        }
        if (*abort_flag) {
          int never = 0;
          for (int j = issued - 1; j >= 0 && j >= issued - WS; --j)
            mbar_wait_bounded(&bar->wfull[j % WS], (uint32_t)(j / WS) & 1u, &never,
                              kDrainLimitNs);
        }
      }
    }
    __syncwarp();  // the whole warp reaches the cluster barrier below together
  } else if (warp == 1) {
    // ---------------- pair MMA issuer (even CTA) ----------------
    if (even) {
      const uint32_t idesc = idesc_f16_f32(2 * BW, BT);
      bool ok = true;
      int g = 0, it = 0;
      for (; it < NT && ok; ++it) {
        if (it > 0) {
          // the previous tile's accumulator has been read out by every group
          // warp of both CTAs
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar->dempty, (uint32_t)(it - 1) & 1u,
                                                         abort_flag, kWaitLimitNs));
          if (!ok) break;
          tc_fence_after();
        }
        for (int kb = 0; kb < KB; ++kb, ++g) {
          const int s = g % XS, a = g % AS;
          ok = __all_sync(0xffffffffu,
                          mbar_wait_bounded(&bar->xfull[s], (uint32_t)(g / XS) & 1u, abort_flag,
                                            kWaitLimitNs) &&
                              mbar_wait_bounded(&bar->afull[a], (uint32_t)(g / AS) & 1u,
                                                abort_flag, kWaitLimitNs));
          if (!ok) break;
          tc_fence_after();
          const uint64_t b_desc0 = smem_desc_sw128(smem_u32(xs + s * L::X_STAGE_BYTES));
          const uint32_t a_base = tmem + A_COL + a * A_STAGE_COLS;
          // k16 steps: those holding k below K, or a LoRA stage's 32 ranks
          const int nk = kb >= KW ? LORA_R / 16 : (kb * BK + 64 < K ? BK / 16 : 4);
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              if (kk < nk)
                mma_f16_ts_pair(tmem + D_COL, a_base + kk * 8,
                                b_desc0 + (uint64_t)(((kk >> 2) * L::X_HALF_BYTES +
                                                      (kk & 3) * 32) >> 4),
                                idesc, (kb | kk) != 0 ? 1u : 0u);
            mma_commit_pair(&bar->xempty[s], kPairMask);
            mma_commit_pair(&bar->aempty[a], kPairMask);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) mma_commit_pair(&bar->dfull, kPairMask);  // tile done
        __syncwarp();
      }
      if (!ok) {
        if (lane == 0) record_timeout(err, bar);
        // wait for the MMAs already issued before anyone frees TMEM
        if (elect_one()) mma_commit_pair(&bar->dfull, kPairMask);
        __syncwarp();
        int never = 0;
        mbar_wait_bounded(&bar->dfull, (uint32_t)it & 1u, &never, kDrainLimitNs);
      }
    }
    __syncwarp();  // the whole warp reaches the cluster barrier below together
  } else {
    // ---------------- dequantisation and accumulator read-out ----------------
    const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
    const int grp = (warp - DQ_WARP0) >> 2;  // stages g = grp mod DQ_GROUPS
    const uint32_t lane_addr = (uint32_t)(32 * quarter) << 16;
    const int col = 32 * quarter + lane;     // this thread's column in the tile
    const int j = grp;                       // this group's A slot
    // this thread's column in weight slot 0 (slot jw adds jw * W_STAGE_BYTES)
    const uint8_t* qw0 = smem + L::W_OFF + col * 4;
    const uint8_t* sc0 = smem + L::W_OFF + QW_STAGE_BYTES + col * 2;
    // this thread's packed zero word in weight slot 0 (eight columns per word)
    const uint8_t* zr0 = smem + L::W_OFF + Z_OFF + (col / 8) * 4;
    const uint32_t zshift = 4u * (uint32_t)(col % 8);
    uint8_t* ystage = smem + L::Y_OFF + grp * L::Y_GROUP_BYTES + quarter * L::Y_WARP_BYTES;

    // Reads out tile d's accumulator (this warp's 32 lanes x its group's TPG
    // tokens), hands it back to the MMA warp, and stores the FP16 values to
    // Y through this warp's staging block.  False if the wait expired.
    auto drain = [&](int d) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait_bounded<true>(&bar->dfull, (uint32_t)d & 1u,
                                                           abort_flag, kWaitLimitNs)))
        return false;
      tc_fence_after();
      uint32_t v0[32], v1[32];
      tmem_ld_32x32b_x32(tmem + lane_addr + D_COL + grp * TPG, v0);
      if constexpr (TPG == 64) tmem_ld_32x32b_x32(tmem + lane_addr + D_COL + grp * TPG + 32, v1);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(dempty_even);  // the MMAs may overwrite it now
      int dn0, dt0;
      walk.coords(d, BT, rank, dn0, dt0);
      if (lane == 0) bulk_wait_read_all();  // the block's previous store has read it
      __syncwarp();
      uint16_t* ys = reinterpret_cast<uint16_t*>(ystage);
#pragma unroll
      for (int q = 0; q < 32; ++q)
        ys[q * 32 + lane] = __half_as_ushort(__float2half_rn(__uint_as_float(v0[q])));
      if constexpr (TPG == 64) {
#pragma unroll
        for (int q = 0; q < 32; ++q)
          ys[(32 + q) * 32 + lane] = __half_as_ushort(__float2half_rn(__uint_as_float(v1[q])));
      }
      fence_proxy_async_smem();  // the staging writes are visible to the store
      __syncwarp();
      const int c0 = dn0 + 32 * quarter, tok0 = dt0 + grp * TPG;
      if (lane == 0 && c0 < N && tok0 < M) {
        tma_store_2d(&y_map, ystage, c0, tok0);
        bulk_commit_group();
      }
      return true;
    };

    bool ok = true;
    int drained = 0;  // tiles whose accumulator this warp has read out
    for (int g = grp; g < G; g += DQ_GROUPS) {
      // Read out every finished tile before this stage.  One must be read
      // out first if this stage's A slot was last used by a later tile, whose
      // MMAs wait for the accumulator.
      const int it = g / KB;
      while (drained < it) {
        const bool forced = g - AS >= (drained + 1) * KB;
        const bool done = __shfl_sync(
            0xffffffffu, (int)mbar_test_wait(smem_u32(&bar->dfull), (uint32_t)drained & 1u), 0);
        if (!forced && !done) break;
        ok = drain(drained);
        if (!ok) break;
        ++drained;
      }
      if (!ok) {
        if (lane == 0) record_timeout(err, bar);
        break;
      }
      const uint32_t ph = (uint32_t)(g / DQ_GROUPS) & 1u;  // A slot phase
      const int jw = g % WS;                                // weight slot
      const uint32_t pw = (uint32_t)(g / WS) & 1u;
      const uint8_t* qw = qw0 + jw * W_STAGE_BYTES;
      const uint8_t* sc = sc0 + jw * W_STAGE_BYTES;
      // qweight and scale tiles of the stage have landed
      ok = __all_sync(0xffffffffu,
                      mbar_wait_bounded<true>(&bar->wfull[jw], pw, abort_flag, kWaitLimitNs));
      if (!ok) {
        if (lane == 0) record_timeout(err, bar);
        break;
      }
      if (g - it * KB >= KW) {
        // LoRA stage: this column's 32 lora_b values, copied as they are
        // (pairs of ranks per 32-bit cell, as the dequantised weights)
        const uint4* brow = reinterpret_cast<const uint4*>(smem + L::W_OFF + jw * W_STAGE_BYTES +
                                                           col * (LORA_R * 2));
        uint32_t cells[LORA_R / 2];
#pragma unroll
        for (int v = 0; v < LORA_R / 8; ++v) {
          const uint4 q = brow[v];
          cells[4 * v] = q.x;
          cells[4 * v + 1] = q.y;
          cells[4 * v + 2] = q.z;
          cells[4 * v + 3] = q.w;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->wempty[jw]);
        ok = __all_sync(0xffffffffu, mbar_wait_bounded<true>(&bar->aempty[j], ph ^ 1u,
                                                             abort_flag, kWaitLimitNs));
        if (!ok) {
          if (lane == 0) record_timeout(err, bar);
          break;
        }
        tc_fence_after();
        tmem_st_32x32b_x16(tmem + lane_addr + A_COL + j * A_STAGE_COLS, cells);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(afull_even + 8u * (uint32_t)j);
        continue;
      }
      // the stage's 16 packed rows, one 64-k half (32 TMEM columns) at a time
      uint32_t cells[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int r8 = 0; r8 < 8; ++r8) {
          const int r = 8 * h + r8;
          // scale row of packed row r inside the stage (0 unless the group is
          // smaller than the 128-k stage)
          const int gl = group_shift >= 7 ? 0 : (r * 8) >> group_shift;
          const uint16_t sv = *reinterpret_cast<const uint16_t*>(sc + gl * S_ROW_BYTES);
          const uint32_t w = *reinterpret_cast<const uint32_t*>(qw + r * (BW * 4));
          uint32_t nat[4];
          if constexpr (ASYM) {
            const uint32_t z = (*reinterpret_cast<const uint32_t*>(
                                    zr0 + jw * W_STAGE_BYTES + gl * Z_ROW_BYTES) >> zshift) & 0xFu;
            dequant_word_natural_z(w, half2_broadcast(sv), zero_sub_low(z), zero_add_high(z), nat);
          } else {
            dequant_word_natural(w, half2_broadcast(sv), nat);
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) cells[4 * r8 + q] = nat[q];
        }
        if (h == 0) {
          // the A slot is free once the pair MMAs of its previous use completed
          ok = __all_sync(0xffffffffu, mbar_wait_bounded<true>(&bar->aempty[j], ph ^ 1u,
                                                               abort_flag, kWaitLimitNs));
          if (!ok) break;
          tc_fence_after();
        } else {
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar->wempty[jw]);  // weight tiles of the stage read
        }
        tmem_st_32x32b_x32(tmem + lane_addr + A_COL + j * A_STAGE_COLS + 32 * h, cells);
      }
      if (!ok) {
        if (lane == 0) record_timeout(err, bar);
        break;
      }
      tmem_wait_st();  // the whole warp's cells are in TMEM
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(afull_even + 8u * (uint32_t)j);
    }
    // the tiles not read out yet
    while (ok && drained < NT) {
      ok = drain(drained);
      if (!ok && lane == 0) record_timeout(err, bar);
      ++drained;
    }
    if (lane == 0) bulk_wait_all();  // this warp's stores have completed
    __syncwarp();
  }

  // neither CTA leaves (or frees TMEM) while the pair's MMAs, loads or
  // signals may still touch it
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

template <int BT, bool ASYM>
cudaError_t launch_pair_t(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                          const int32_t* qzeros, uint16_t* y, int64_t M, int64_t K, int64_t N,
                          int group_shift, int scale_rows, int64_t n_groups, const uint16_t* t,
                          const uint16_t* lora_b, int64_t rank, cudaStream_t stream,
                          const DeviceInfo& dev) {
  using L = PairLayout<BT>;
  CUtensorMap x_map, qw_map, s_map, y_map, t_map, b_map, qz_map;
  // X as [K/64][M][64] (one copy of both 64-k halves per stage) when K is a
  // multiple of 64, else as [M][K] (one copy per half); rows at or beyond M
  // and k at or beyond K read as zero either way
  int x3d = 0;
  if (K % 64 == 0) {
    const uint64_t dims[3] = {64, (uint64_t)M, (uint64_t)(K / 64)};
    const uint64_t strides[2] = {(uint64_t)K * 2, 128};
    const uint32_t box[3] = {64, (uint32_t)L::HT, 2};
    x3d = tensor_map_3d(&x_map, x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_128B) ? 1 : 0;
  }
  if ((!x3d && !tensor_map_2d(&x_map, x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)K,
                              (uint64_t)M, (uint64_t)K * 2, 64, L::HT,
                              CU_TENSOR_MAP_SWIZZLE_128B)) ||
      !tensor_map_2d(&qw_map, qweight, CU_TENSOR_MAP_DATA_TYPE_INT32, (uint64_t)N,
                     (uint64_t)(K / 8), (uint64_t)N * 4, BW, BK / 8, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !tensor_map_2d(&s_map, scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, (uint64_t)N,
                     (uint64_t)n_groups, (uint64_t)N * 2, BW, (uint32_t)scale_rows,
                     CU_TENSOR_MAP_SWIZZLE_NONE) ||
      // Y blocks of 32 columns x BT/4 tokens, one per dequantisation warp
      !tensor_map_2d(&y_map, y, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)N, (uint64_t)M,
                     (uint64_t)N * 2, 32, L::TPG, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (ASYM) {
    // zero points [n_groups, N/8] int32: 16 words (128 columns) x the stage's rows
    if (!tensor_map_2d(&qz_map, qzeros, CU_TENSOR_MAP_DATA_TYPE_INT32, (uint64_t)(N / 8),
                       (uint64_t)n_groups, (uint64_t)(N / 8) * 4, BW / 8, (uint32_t)scale_rows,
                       CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  } else {
    qz_map = qw_map;  // not read for symmetric weights
  }
  int lora_stages = 0;
  if (rank > 0) {
    // T [M, rank]: 64 columns x BT/2 rows per copy (128-byte swizzle, the
    // B operand); lora_b [N, rank]: 32 columns x 128 rows (plain rows)
    if (!tensor_map_2d(&t_map, t, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)rank, (uint64_t)M,
                       (uint64_t)rank * 2, 64, L::HT, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tensor_map_2d(&b_map, lora_b, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)rank,
                       (uint64_t)N, (uint64_t)rank * 2, LORA_R, BW, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    lora_stages = (int)((rank + LORA_R - 1) / LORA_R);
  } else {
    t_map = x_map;  // not read without an adapter
    b_map = qw_map;
  }
  constexpr size_t smem = L::kSmemBytes;
  static std::once_flag attr_once[64];
  static cudaError_t attr_err[64];
  const int d = dev.device & 63;
  std::call_once(attr_once[d], [&] {
    attr_err[d] = cudaFuncSetAttribute(prefill_pair_kernel<BT, ASYM>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  });
  if (attr_err[d] != cudaSuccess) return attr_err[d];
  // column pairs of 2 x 128 (with an odd count of 128-column tiles the last
  // pair's odd CTA has no columns: it loads no weights and stores nothing)
  const int64_t n_pairs = ((N + BW - 1) / BW + 1) / 2;
  const int64_t tiles = n_pairs * ((M + BT - 1) / BT);
  const int64_t clusters = std::min<int64_t>(tiles, std::max(1, dev.num_sms / 2));
  // With an adapter this launch may start while the one computing T still
  // runs (only the first read of T waits for it); the weights and X do not
  // depend on that launch.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = lora_stages > 0 ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, prefill_pair_kernel<BT, ASYM>, x_map, qw_map, s_map, qz_map,
                            y_map, t_map, b_map, (int)M, (int)K, (int)N, group_shift, scale_rows,
                            x3d, (int)n_pairs, (int)tiles, lora_stages, dev.error_word);
}

// Both pair tiles, symmetric or with zero points, with or without an adapter.
cudaError_t launch_pair(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                        const int32_t* qzeros, uint16_t* y, int64_t M, int64_t K, int64_t N,
                        int group_shift, const uint16_t* t, const uint16_t* lora_b, int64_t rank,
                        cudaStream_t stream, const DeviceInfo& dev) {
  const int64_t n_groups = (group_shift == 62 || (int64_t(1) << group_shift) >= K)
                               ? 1 : (K + (int64_t(1) << group_shift) - 1) >> group_shift;
  const int scale_rows = group_shift >= 7 ? 1 : (BK >> group_shift);
  if (qzeros) {
    if (M <= 128)
      return launch_pair_t<128, true>(x, qweight, scales, qzeros, y, M, K, N, group_shift,
                                      scale_rows, n_groups, t, lora_b, rank, stream, dev);
    return launch_pair_t<256, true>(x, qweight, scales, qzeros, y, M, K, N, group_shift,
                                    scale_rows, n_groups, t, lora_b, rank, stream, dev);
  }
  if (M <= 128)
    return launch_pair_t<128, false>(x, qweight, scales, nullptr, y, M, K, N, group_shift,
                                     scale_rows, n_groups, t, lora_b, rank, stream, dev);
  return launch_pair_t<256, false>(x, qweight, scales, nullptr, y, M, K, N, group_shift,
                                   scale_rows, n_groups, t, lora_b, rank, stream, dev);
}

}  // namespace

cudaError_t launch_prefill_pair_lora(const uint16_t* x, const int32_t* qweight,
                                     const uint16_t* scales, uint16_t* y, int64_t M, int64_t K,
                                     int64_t N, int group_shift, const uint16_t* t,
                                     const uint16_t* lora_b, int64_t rank, cudaStream_t stream,
                                     const DeviceInfo& dev) {
  return launch_pair(x, qweight, scales, nullptr, y, M, K, N, group_shift, t, lora_b, rank,
                     stream, dev);
}

cudaError_t launch_prefill_pair_asym(const uint16_t* x, const int32_t* qweight,
                                     const uint16_t* scales, const int32_t* qzeros, uint16_t* y,
                                     int64_t M, int64_t K, int64_t N, int group_shift,
                                     cudaStream_t stream, const DeviceInfo& dev) {
  return launch_pair(x, qweight, scales, qzeros, y, M, K, N, group_shift, nullptr, nullptr, 0,
                     stream, dev);
}

cudaError_t launch_prefill_pair(const uint16_t* x, const int32_t* qweight,
                                const uint16_t* scales, uint16_t* y, int64_t M, int64_t K,
                                int64_t N, int group_shift, cudaStream_t stream,
                                const DeviceInfo& dev) {
  return launch_pair(x, qweight, scales, nullptr, y, M, K, N, group_shift, nullptr, nullptr, 0,
                     stream, dev);
}

}  // namespace gptq
