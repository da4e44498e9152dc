// W[K, N] = fp16((q - 8) * s): the dequantisation entry (gptq_dequant).
//
// Operation: GPTQ-Pro README, "Runtime contract" (symmetric INT4 GPTQ, native
// int32 qweight, FP16); each weight is rounded once from the exact product.
//
// One thread handles one packed row i (eight k) by eight columns: two 16-byte
// qweight loads, one 16-byte scale load, eight 16-byte stores (one per k).
// A warp therefore reads 1 KiB of qweight and writes 32 rows x 256 B, all
// coalesced.  HBM-bound: 2.5 bytes of traffic per weight (0.5 read, 2 written).
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace gptq {

__global__ void __launch_bounds__(256) dequant_kernel(const int32_t* __restrict__ qweight,
                                                      const uint16_t* __restrict__ scales,
                                                      uint16_t* __restrict__ w_out, int64_t K,
                                                      int64_t N, int group_shift) {
  const int64_t cols8 = N / 8;
  const int64_t total = (K / 8) * cols8;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = t / cols8;          // packed row
    const int64_t n0 = (t - i * cols8) * 8;
    const int64_t g = (i * 8) >> group_shift;
    const uint4 qa = ld_stream_v4(qweight + i * N + n0);
    const uint4 qb = ld_stream_v4(qweight + i * N + n0 + 4);
    const uint4 sv = ld_nc_v4(scales + g * N + n0);
    const uint32_t words[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
    const uint32_t sp[4] = {sv.x, sv.y, sv.z, sv.w};
    uint32_t p[8][4];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint16_t s = (c & 1) ? (uint16_t)(sp[c >> 1] >> 16) : (uint16_t)(sp[c >> 1] & 0xFFFF);
      dequant_word_paired(words[c], half2_broadcast(s), p[c]);
    }
    uint16_t* out = w_out + (i * 8) * N + n0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint4 lo, hi;  // row k_j and row k_{j+4}, eight columns each
      lo.x = prmt(p[0][j], p[1][j], 0x5410);
      lo.y = prmt(p[2][j], p[3][j], 0x5410);
      lo.z = prmt(p[4][j], p[5][j], 0x5410);
      lo.w = prmt(p[6][j], p[7][j], 0x5410);
      hi.x = prmt(p[0][j], p[1][j], 0x7632);
      hi.y = prmt(p[2][j], p[3][j], 0x7632);
      hi.z = prmt(p[4][j], p[5][j], 0x7632);
      hi.w = prmt(p[6][j], p[7][j], 0x7632);
      *reinterpret_cast<uint4*>(out + j * N) = lo;
      *reinterpret_cast<uint4*>(out + (j + 4) * N) = hi;
    }
  }
}

cudaError_t launch_dequant(const int32_t* qweight, const uint16_t* scales, int64_t K, int64_t N,
                           int group_shift, uint16_t* w_out, cudaStream_t stream,
                           const DeviceInfo& dev) {
  const int64_t total = (K / 8) * (N / 8);
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  const int64_t cap = (int64_t)dev.num_sms * 8;
  if (blocks > cap) blocks = cap;
  dequant_kernel<<<(unsigned)blocks, threads, 0, stream>>>(qweight, scales, w_out, K, N,
                                                           group_shift);
  return cudaGetLastError();
}

}  // namespace gptq
