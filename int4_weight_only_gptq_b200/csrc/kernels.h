// Internal interface between the C ABI (api.cu) and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gptq {

struct DeviceInfo {
  int device = -1;
  int num_sms = 0;
  int cc_major = 0;
  int cc_minor = 0;
  int smem_optin = 0;   // max dynamic shared memory per block (opt-in)
  int l2_bytes = 0;
  int* error_word = nullptr;  // device address of this device's error word
  uint16_t* lora_scratch = nullptr;  // device address of the static T buffer
  unsigned long long* t_flags = nullptr;  // device address of the T hand-over flags
};

// Slots of the flags through which the CTAs computing a LoRA adapter's T
// inside the layer's launch hand it over (one slot per call, reused after
// this many calls on the device).
constexpr int kTFlagSlots = 1024;

// Error codes written to the device error word (match gptq_status values).
constexpr int kDeviceErrTimeout = 7;
constexpr int kDeviceErrIndex = 10;  // a g_idx entry outside 0 .. n_groups - 1

// log2(group), or 62 for group == -1 (then (8*i) >> 62 == 0 for every row).
inline int group_shift_of(int32_t group) {
  if (group == -1) return 62;
  int s = 0;
  while ((1 << s) < group) ++s;
  return s;
}

cudaError_t launch_dequant(const int32_t* qweight, const uint16_t* scales, int64_t K, int64_t N,
                           int group_shift, uint16_t* w_out, cudaStream_t stream,
                           const DeviceInfo& dev);

// Decode (M <= 64).  splits = number of CTAs that share one column block along
// K (the cluster size, 1..8); 0 picks it from the shape.
int decode_pick_splits(int64_t M, int64_t K, int64_t N, bool lora, const DeviceInfo& dev);
// Packed rows per ring stage of a decode launch (64: 512 k, 32: 256 k) for M
// tokens over nblk column blocks; splits = 0 when the launch picks it.
int decode_stage_rows(int64_t M, int64_t nblk, int64_t K, int splits, bool lora,
                      const DeviceInfo& dev);
int decode_pick_splits_blocks(int64_t column_blocks, int64_t K, int prs, const DeviceInfo& dev);
cudaError_t launch_decode(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                          uint16_t* y, int64_t M, int64_t K, int64_t N, int group_shift,
                          int splits, cudaStream_t stream, const DeviceInfo& dev);
// Decode with asymmetric zero points: qzeros [n_groups, N/8] int32, eight
// 4-bit zeros per word along N (N % 32 == 0).
cudaError_t launch_decode_asym(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                               const int32_t* qzeros, uint16_t* y, int64_t M, int64_t K,
                               int64_t N, int group_shift, cudaStream_t stream,
                               const DeviceInfo& dev);
// Decode with a LoRA adapter: t = fp16(x . lora_a^T) [M, rank] (from
// launch_lora_down), lora_b [N, rank]; rank/128 extra stages in the last
// split of each column block.
// The adapter's T computed inside the layer's decode launch (on CTAs beside
// the column blocks) when the SMs that launch leaves free allow it; false if
// the two-launch form must be used (then nothing is enqueued).
bool decode_lora_fused_fits(int64_t M, int64_t K, int64_t N, int64_t rank, const DeviceInfo& dev);
cudaError_t launch_decode_lora_fused(const uint16_t* x, const int32_t* qweight,
                                     const uint16_t* scales, uint16_t* y, int64_t M, int64_t K,
                                     int64_t N, int group_shift, uint16_t* t,
                                     const uint16_t* lora_a, const uint16_t* lora_b,
                                     int64_t rank, cudaStream_t stream, const DeviceInfo& dev);
cudaError_t launch_decode_lora(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                               uint16_t* y, int64_t M, int64_t K, int64_t N, int group_shift,
                               const uint16_t* t, const uint16_t* lora_b, int64_t rank,
                               cudaStream_t stream, const DeviceInfo& dev);
// Decode of `count` linears that share X (1..GPTQ_MAX_GROUPED), one launch;
// the split is picked from the total number of column blocks.
// Act order: W[k,n] = fp16((q[k,n] - 8) * scales[g_idx[k], n]), g_idx [K]
// int32, scales [n_groups, N]; any M (tiles of at most 64 tokens).
cudaError_t launch_decode_gidx(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                               const int32_t* g_idx, uint16_t* y, int64_t M, int64_t K,
                               int64_t N, int64_t n_groups, cudaStream_t stream,
                               const DeviceInfo& dev);
cudaError_t launch_decode_grouped(const uint16_t* x, const int32_t* const* qweights,
                                  const uint16_t* const* scales, const int64_t* ns,
                                  uint16_t* const* ys, int count, int64_t M, int64_t K,
                                  int group_shift, cudaStream_t stream, const DeviceInfo& dev);

// Prefill (any M >= 1): TMA + tcgen05 with TMEM accumulators.
cudaError_t launch_prefill(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                           uint16_t* y, int64_t M, int64_t K, int64_t N, int group_shift,
                           cudaStream_t stream, const DeviceInfo& dev);
// The same on CTA pairs (tcgen05 cta_group::2; 256 weight columns x 128 or
// 256 tokens per pair, half of the X tile loaded by each CTA).
cudaError_t launch_prefill_pair(const uint16_t* x, const int32_t* qweight,
                                const uint16_t* scales, uint16_t* y, int64_t M, int64_t K,
                                int64_t N, int group_shift, cudaStream_t stream,
                                const DeviceInfo& dev);
// The same with a LoRA adapter: t = fp16(x . lora_a^T) [M, rank] (from
// launch_lora_down), lora_b [N, rank]; T . lora_b^T is added to the
// accumulator as rank/32 extra stages per tile.
cudaError_t launch_prefill_pair_lora(const uint16_t* x, const int32_t* qweight,
                                     const uint16_t* scales, uint16_t* y, int64_t M, int64_t K,
                                     int64_t N, int group_shift, const uint16_t* t,
                                     const uint16_t* lora_b, int64_t rank, cudaStream_t stream,
                                     const DeviceInfo& dev);
// The pair kernel with asymmetric zero points: qzeros [n_groups, N/8] int32,
// eight 4-bit zeros per word along N (N % 32 == 0).
cudaError_t launch_prefill_pair_asym(const uint16_t* x, const int32_t* qweight,
                                     const uint16_t* scales, const int32_t* qzeros, uint16_t* y,
                                     int64_t M, int64_t K, int64_t N, int group_shift,
                                     cudaStream_t stream, const DeviceInfo& dev);
// t [M, r] = fp16(x . lora_a^T), lora_a [r, K] (the adapter's down-projection).
// free_sms: SMs that the layer's launch after it leaves unused (0 if none or
// unknown); up to 32 tokens the launch stays on them when it can.
cudaError_t launch_lora_down(const uint16_t* x, const uint16_t* lora_a, uint16_t* t, int64_t M,
                             int64_t K, int64_t r, int free_sms, cudaStream_t stream,
                             const DeviceInfo& dev);
// CTAs of one decode launch of this shape (column blocks x K split).
int64_t decode_ctas(int64_t M, int64_t K, int64_t N, bool lora, const DeviceInfo& dev);

}  // namespace gptq
