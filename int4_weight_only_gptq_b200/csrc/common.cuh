// Device helpers shared by the sm_100a kernels of the W4A16 GPTQ library.
//
// The dequantisation primitive follows the layer's definition exactly
// (GPTQ-Pro README, "Runtime contract": symmetric INT4, zero point 8, FP16):
// a code q becomes the FP16 value 1024 + q by OR-ing it into the mantissa of
// 1024.0 (exponent bits 0x6400), (1024 + q) - 1032 = q - 8 is exact, and the
// product (q - 8) * s is rounded once to FP16 (round to nearest even).  The
// arithmetic is written with explicit .rn modifiers so that the compiler cannot
// contract it into a fused multiply-add with a different rounding.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace gptq {

constexpr uint32_t kMagic1024 = 0x64006400u;   // half2(1024, 1024)
constexpr uint32_t kMinus1032 = 0x64086408u;   // half2(1032, 1032) (subtracted)
constexpr uint32_t kOneSixteenth = 0x2C002C00u; // half2(1/16, 1/16)
constexpr uint32_t kMinus72 = 0xD480D480u;      // half2(-72, -72)

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;  // (a & b) | c
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

__device__ __forceinline__ uint32_t hsub2_rn(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t hmul2_rn(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t hfma2_rn(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// Eight codes of one qweight word -> four half2 (q - 8), paired (k, k+4):
//   p[0] = (k0, k4), p[1] = (k1, k5), p[2] = (k2, k6), p[3] = (k3, k7)
// (low half first).  All four are exact small integers.
__device__ __forceinline__ void unpack_centered(uint32_t w, uint32_t p[4]) {
  const uint32_t w8 = w >> 8;  // logical shift: the word is unsigned here
  p[0] = hsub2_rn(lop3_and_or(w, 0x000F000Fu, kMagic1024), kMinus1032);
  p[1] = hfma2_rn(lop3_and_or(w, 0x00F000F0u, kMagic1024), kOneSixteenth, kMinus72);
  p[2] = hsub2_rn(lop3_and_or(w8, 0x000F000Fu, kMagic1024), kMinus1032);
  p[3] = hfma2_rn(lop3_and_or(w8, 0x00F000F0u, kMagic1024), kOneSixteenth, kMinus72);
}

// Dequantised weights of one word, paired (k, k+4) as above: one rounding.
__device__ __forceinline__ void dequant_word_paired(uint32_t w, uint32_t s2, uint32_t p[4]) {
  unpack_centered(w, p);
#pragma unroll
  for (int j = 0; j < 4; ++j) p[j] = hmul2_rn(p[j], s2);
}

// sm += the FP32 dot product of eight FP16 x (one 16-byte chunk) with eight
// weights already widened to four float2, in k order.
__device__ __forceinline__ void fma8(float& sm, const uint4 xv, const float2 a0, const float2 a1,
                                     const float2 a2, const float2 a3) {
  const float2 x0 = __half22float2(*reinterpret_cast<const __half2*>(&xv.x));
  const float2 x1 = __half22float2(*reinterpret_cast<const __half2*>(&xv.y));
  const float2 x2 = __half22float2(*reinterpret_cast<const __half2*>(&xv.z));
  const float2 x3 = __half22float2(*reinterpret_cast<const __half2*>(&xv.w));
  sm = fmaf(x0.x, a0.x, sm);
  sm = fmaf(x0.y, a0.y, sm);
  sm = fmaf(x1.x, a1.x, sm);
  sm = fmaf(x1.y, a1.y, sm);
  sm = fmaf(x2.x, a2.x, sm);
  sm = fmaf(x2.y, a2.y, sm);
  sm = fmaf(x3.x, a3.x, sm);
  sm = fmaf(x3.y, a3.y, sm);
}

// Dequantised weights of one word with a scale per pair (act-order weights,
// whose k can each take a different group): s2[j] holds the scales of k_j
// (low half) and k_{j+4} (high half).  One rounding per weight, as above.
__device__ __forceinline__ void dequant_word_paired_per_pair(uint32_t w, const uint32_t s2[4],
                                                             uint32_t p[4]) {
  unpack_centered(w, p);
#pragma unroll
  for (int j = 0; j < 4; ++j) p[j] = hmul2_rn(p[j], s2[j]);
}

// The same four half2 for a scale with |s| < 2^-4, with two FP16 operations
// fewer.  Codes at bits 4..7 of each 16-bit half, masked out of the word, are
// the FP16 subnormals q * 2^-20; one fused multiply-add with b2 = s * 2^20 and
// c2 = -8 s computes q * s - 8 s = (q - 8) * s exactly and rounds it once, the
// same value as the subtract-then-multiply of dequant_word_paired.  b2 and c2
// are exact (scaling by powers of two), and b2 stays finite because |s| < 2^-4.
// Pairs (k1, k5) and (k3, k7) take this form; (k0, k4) and (k2, k6) keep the
// magic-number form, which balances the FP16 and integer pipes.  Only for
// 0 < s < 2^-4: with s <= 0 the sum q * s - 8 s can give +0 where the
// definition's product gives -0.
__device__ __forceinline__ bool scale_fits_subnormal_form(uint32_t s2) {
  return (s2 & 0xFFFFu) - 1u < 0x2BFFu;  // the low half's bits in 0x0001 .. 0x2BFF
}

__device__ __forceinline__ void subnormal_form_constants(uint32_t s2, uint32_t& b2, uint32_t& c2) {
  constexpr uint32_t k1024 = 0x64006400u;     // half2(1024, 1024)
  constexpr uint32_t kMinus8 = 0xC800C800u;   // half2(-8, -8)
  b2 = hmul2_rn(hmul2_rn(s2, k1024), k1024);  // s * 2^20, exact
  c2 = hmul2_rn(s2, kMinus8);                 // -8 s, exact
}

__device__ __forceinline__ uint32_t and_b32(uint32_t a, uint32_t m) {
  uint32_t r;
  asm("and.b32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(m));
  return r;
}

__device__ __forceinline__ void dequant_word_paired_small_scale(uint32_t w, uint32_t s2,
                                                                uint32_t b2, uint32_t c2,
                                                                uint32_t p[4]) {
  const uint32_t w8 = w >> 8;
  p[0] = hmul2_rn(hsub2_rn(lop3_and_or(w, 0x000F000Fu, kMagic1024), kMinus1032), s2);
  p[1] = hfma2_rn(and_b32(w, 0x00F000F0u), b2, c2);
  p[2] = hmul2_rn(hsub2_rn(lop3_and_or(w8, 0x000F000Fu, kMagic1024), kMinus1032), s2);
  p[3] = hfma2_rn(and_b32(w8, 0x00F000F0u), b2, c2);
}

// Same, in natural k order: n[j] = (k_{2j}, k_{2j+1}).
__device__ __forceinline__ void dequant_word_natural(uint32_t w, uint32_t s2, uint32_t n[4]) {
  uint32_t p[4];
  dequant_word_paired(w, s2, p);
  n[0] = prmt(p[0], p[1], 0x5410);  // (k0, k1)
  n[1] = prmt(p[2], p[3], 0x5410);  // (k2, k3)
  n[2] = prmt(p[0], p[1], 0x7632);  // (k4, k5)
  n[3] = prmt(p[2], p[3], 0x7632);  // (k6, k7)
}

// With a zero point z (0..15) per weight instead of the constant 8: the
// subtrahends are half2(1024 + z) for the low nibble pairs and the addends
// half2(-(64 + z)) for the high pairs (bit patterns 0x6400 + z and
// 0xD400 + 16 z), so every value q - z (in -15..15) is again exact and the
// scale multiply rounds once.  z = 8 gives the constants of unpack_centered.
__device__ __forceinline__ uint32_t zero_sub_low(uint32_t z) {
  const uint32_t h = 0x6400u + z;
  return h | (h << 16);
}
__device__ __forceinline__ uint32_t zero_add_high(uint32_t z) {
  const uint32_t h = 0xD400u + 16u * z;
  return h | (h << 16);
}

// dequant_word_paired with the zero point given as those two constants.
__device__ __forceinline__ void dequant_word_paired_z(uint32_t w, uint32_t s2, uint32_t zlo,
                                                      uint32_t zhi, uint32_t p[4]) {
  const uint32_t w8 = w >> 8;
  p[0] = hmul2_rn(hsub2_rn(lop3_and_or(w, 0x000F000Fu, kMagic1024), zlo), s2);
  p[1] = hmul2_rn(hfma2_rn(lop3_and_or(w, 0x00F000F0u, kMagic1024), kOneSixteenth, zhi), s2);
  p[2] = hmul2_rn(hsub2_rn(lop3_and_or(w8, 0x000F000Fu, kMagic1024), zlo), s2);
  p[3] = hmul2_rn(hfma2_rn(lop3_and_or(w8, 0x00F000F0u, kMagic1024), kOneSixteenth, zhi), s2);
}

// dequant_word_natural with the zero point given as those two constants.
__device__ __forceinline__ void dequant_word_natural_z(uint32_t w, uint32_t s2, uint32_t zlo,
                                                       uint32_t zhi, uint32_t n[4]) {
  const uint32_t w8 = w >> 8;
  uint32_t p[4];
  p[0] = hmul2_rn(hsub2_rn(lop3_and_or(w, 0x000F000Fu, kMagic1024), zlo), s2);
  p[1] = hmul2_rn(hfma2_rn(lop3_and_or(w, 0x00F000F0u, kMagic1024), kOneSixteenth, zhi), s2);
  p[2] = hmul2_rn(hsub2_rn(lop3_and_or(w8, 0x000F000Fu, kMagic1024), zlo), s2);
  p[3] = hmul2_rn(hfma2_rn(lop3_and_or(w8, 0x00F000F0u, kMagic1024), kOneSixteenth, zhi), s2);
  n[0] = prmt(p[0], p[1], 0x5410);  // (k0, k1)
  n[1] = prmt(p[2], p[3], 0x5410);  // (k2, k3)
  n[2] = prmt(p[0], p[1], 0x7632);  // (k4, k5)
  n[3] = prmt(p[2], p[3], 0x7632);  // (k6, k7)
}

__device__ __forceinline__ uint32_t half2_broadcast(uint16_t h) {
  return (uint32_t)h | ((uint32_t)h << 16);
}

// ---- global loads ----------------------------------------------------------

// Streaming 16-byte load: read-only path, not kept in L1.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// ---- shared memory / cluster ------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Barrier among `count` threads (whole warps) of this CTA on named barrier
// `id` (1..15; 0 is __syncthreads).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Address of the same shared variable in another CTA of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}

__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// ---- mbarrier (bounded waits) ------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Arrive on an mbarrier of any CTA of the cluster (shared::cluster address).
// CTA-scope release: it hands over TMEM contents, whose order is set by the
// tcgen05 wait and fences around the arrive; a cluster-scope release would
// also wait for this thread's memory writes to reach cluster scope, which
// costs thousands of cycles under load and orders nothing the reader needs.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cta.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Has the phase with the given parity completed?  Never waits.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Same, but a thread whose phase has not completed may be suspended for up to
// `hint_ns` nanoseconds (it resumes as soon as the phase completes), so that
// waiting warps do not take issue slots from working ones.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar_addr, uint32_t parity,
                                                    uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

}  // namespace gptq
