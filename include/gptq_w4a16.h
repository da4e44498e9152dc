/*
 * gptq_w4a16.h — C ABI of the B200 (sm_100a) symmetric INT4 GPTQ W4A16 linear.
 *
 *   Y[M,N] = X[M,K] . W[K,N],   W[k,n] = fp16_RNE((q[k,n] - 8) * scales[k/G, n])
 *   q[k,n] = (uint32(qweight[k/8, n]) >> (4*(k%8))) & 0xF
 *
 * Source of the operation: GPTQ-Pro README, "Runtime contract" (symmetric GPTQ
 * INT4, FP16 activations, desc_act=False, native int32 qweight, group sizes
 * -1/16/32/64/128/256/512/1024, input features divisible by 16, output
 * features divisible by 8) and "Ampere kernel architecture" (a small-M fused
 * decode path, a tensor-core prefill path, FP32 accumulation, deterministic
 * split-K; all paths read the original int32 qweight); GPTQModel wiki
 * "Installation and Quickstart", "Defaults and compatibility decisions" (sym
 * True, pack_dtype int32).  The pages do not state the nibble order; this
 * library reads the lowest nibble as the lowest k.
 *
 * Conventions for every entry point:
 *  - Pointers named x, qweight, scales, y, w_out are DEVICE pointers on the
 *    current CUDA device, dense and row-major.  FP16 values travel as their
 *    16-bit patterns (uint16_t).  All must be 16-byte aligned.
 *  - The caller owns every buffer.  The library allocates no device memory,
 *    keeps no dequantised or repacked copy of the weights, and holds no state
 *    between calls other than a per-device attribute cache and a device-side
 *    error word (see gptq_device_error).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *    stream-ordered and asynchronous: they enqueue work and return without
 *    synchronising.
 *  - Arguments are checked before anything is enqueued.  A failed check
 *    returns a gptq_status and enqueues nothing; there is no fallback path.
 *  - Results are deterministic: the same inputs give bitwise-identical outputs.
 *  - The library is reentrant; concurrent calls on different streams are safe.
 */
#ifndef GPTQ_W4A16_H
#define GPTQ_W4A16_H

#include <stdint.h>

#if defined(__GNUC__)
#define GPTQ_API __attribute__((visibility("default")))
#else
#define GPTQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GPTQ_OK = 0,
    GPTQ_ERR_NULL = 1,     /* a required pointer is NULL                              */
    GPTQ_ERR_SHAPE = 2,    /* M < 0, K <= 0, N <= 0, K % 16, N % 8, or a size limit    */
    GPTQ_ERR_GROUP = 3,    /* group not in {-1,16,32,64,128,256,512,1024}              */
    GPTQ_ERR_ALIGN = 4,    /* a pointer is not 16-byte aligned                        */
    GPTQ_ERR_DEVICE = 5,   /* no current device, or it is not compute capability 10.0 */
    GPTQ_ERR_CUDA = 6,     /* the CUDA runtime reported an error at launch             */
    GPTQ_ERR_TIMEOUT = 7,  /* a kernel gave up a bounded wait (see gptq_device_error)  */
    GPTQ_ERR_ALIAS = 8,    /* the output overlaps an input                            */
    GPTQ_ERR_KERNEL = 9,   /* kernel_id names no kernel, or one that cannot take M     */
    GPTQ_ERR_INDEX = 10    /* a g_idx entry outside 0 .. n_groups-1 (device-reported) */
} gptq_status;

/* Kernel identifiers reported by gptq_w4a16_select and accepted by
 * gptq_w4a16_gemm_kernel. */
#define GPTQ_KERNEL_AUTO 0
#define GPTQ_KERNEL_DECODE 1   /* M <= 64: streams qweight, split-K, tcgen05 MMA   */
#define GPTQ_KERNEL_PREFILL 2  /* any M: TMA + tcgen05 MMA with TMEM accumulators  */

/* Size limits (inclusive). */
#define GPTQ_MAX_K 65536
#define GPTQ_MAX_N 1048576
#define GPTQ_MAX_M 8388608
#define GPTQ_DECODE_MAX_M 64
#define GPTQ_LORA_DECODE_MAX_M 32 /* gptq_w4a16_gemm_lora: decode kernel up to here */
#define GPTQ_MAX_GROUPED 8     /* linears per gptq_w4a16_gemm_grouped call */
#define GPTQ_MAX_LORA_RANK 256 /* largest adapter rank of gptq_w4a16_gemm_lora */
#define GPTQ_LORA_SCRATCH_BYTES (8 << 20) /* T buffer of gptq_w4a16_gemm_lora_noalloc */
#define GPTQ_GIDX_MAX_GROUPS 640 /* scale rows of gptq_w4a16_gemm_gidx (a tile per CTA) */

/*
 * Y = X . dequant(qweight, scales).
 *   x       [M, K]          FP16 bits    (may be NULL only when M == 0)
 *   qweight [K/8, N]        int32, eight 4-bit codes along K, lowest nibble = lowest k
 *   scales  [n_groups, N]   FP16 bits, n_groups = 1 if group == -1 or group >= K,
 *                           else ceil(K / group); the last group may be ragged
 *   y       [M, N]          FP16 bits, written (may be NULL only when M == 0);
 *                           must not overlap x, qweight or scales
 * Accumulation is FP32; each output is rounded once to FP16 (nearest-even).
 * M == 0 returns GPTQ_OK and enqueues nothing.  The kernel is chosen by
 * gptq_w4a16_select.
 */
GPTQ_API int gptq_w4a16_gemm(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                    int64_t M, int64_t K, int64_t N, int32_t group,
                    uint16_t* y, void* stream);

/*
 * As gptq_w4a16_gemm, with the kernel forced: kernel_id is one of the
 * GPTQ_KERNEL_* values (AUTO behaves exactly like gptq_w4a16_gemm).  DECODE
 * accepts M <= GPTQ_DECODE_MAX_M only (else GPTQ_ERR_KERNEL).  Meant for tests
 * and benchmarks that compare the kernels on the same shape.
 */
GPTQ_API int gptq_w4a16_gemm_kernel(const uint16_t* x, const int32_t* qweight,
                           const uint16_t* scales, int64_t M, int64_t K, int64_t N,
                           int32_t group, uint16_t* y, void* stream, int32_t kernel_id);

/*
 * As gptq_w4a16_gemm_kernel with GPTQ_KERNEL_DECODE, with the number of CTAs
 * that split K within one column block fixed to `splits` (1..8) instead of
 * chosen from the shape.  Any split gives a correct, deterministic result;
 * the choice only moves performance.  Meant for tuning sweeps and tests.
 */
GPTQ_API int gptq_w4a16_gemm_decode_splits(const uint16_t* x, const int32_t* qweight,
                                           const uint16_t* scales, int64_t M, int64_t K,
                                           int64_t N, int32_t group, uint16_t* y, void* stream,
                                           int32_t splits);

/*
 * Several linears that share one input X, for example the q, k and v
 * projections or the gate and up projections of a layer:
 *   Y_i = X . dequant(qweights[i], scales[i]),   i = 0 .. count-1.
 * The GPTQModel wiki ("Installation and Quickstart") describes engines that
 * merge such linears into one (gate_up_proj, qkv_proj); here each linear keeps
 * its own native qweight and scales, and X is shared.
 *   x          [M, K] FP16 bits, device (may be NULL only when M == 0)
 *   qweights   HOST array of `count` device pointers, qweights[i] [K/8, Ns[i]]
 *   scales     HOST array of `count` device pointers, scales[i] [n_groups, Ns[i]]
 *              (one group size and one K for all linears)
 *   Ns         HOST array of `count` output widths, each > 0 and % 8 == 0
 *   ys         HOST array of `count` device pointers, ys[i] [M, Ns[i]], written;
 *              pairwise disjoint and not overlapping x, any qweight or any scales
 *   count      1 .. GPTQ_MAX_GROUPED
 * For M <= GPTQ_DECODE_MAX_M all linears are computed by ONE decode launch
 * (one X read, one fixed launch cost); for larger M each linear gets its own
 * prefill launch.  The host arrays are read during the call only.  Results
 * are within the same tolerance as separate calls, and deterministic.
 * Errors as gptq_w4a16_gemm (any linear failing a check fails the call before
 * anything is enqueued), plus GPTQ_ERR_SHAPE for count out of range.
 */
GPTQ_API int gptq_w4a16_gemm_grouped(const uint16_t* x, const int32_t* const* qweights,
                                     const uint16_t* const* scales, const int64_t* Ns,
                                     int32_t count, int64_t M, int64_t K, int32_t group,
                                     uint16_t* const* ys, void* stream);

/*
 * The layer with asymmetric zero points (GPTQ's sym=False weights):
 *   Y = X . W,  W[k,n] = fp16((q[k,n] - z[k/G, n]) * scales[k/G, n])
 *   z[g,n] = (uint32(qzeros[g, n/8]) >> 4*(n%8)) & 0xF
 * The GPTQModel wiki ("Installation and Quickstart", "Defaults and
 * compatibility decisions") defaults sym to True and notes that not every
 * backend accepts asymmetric weights; the GPTQ-Pro README puts them outside
 * its contract.  Read with GPTQ's packed zero points, each taken as stored:
 *   qzeros   [n_groups, N/8] int32, device, eight 4-bit zeros per word along
 *            N (lowest nibble = lowest n), 16-byte aligned
 *   N        a multiple of 32 (zero-point rows are copied in 16-byte units)
 * (q - z) is exact and scaled with one rounding, as in the symmetric layer;
 * with every z = 8 the result equals gptq_w4a16_gemm's.  The kernel follows
 * M as in gptq_w4a16_gemm (decode up to GPTQ_DECODE_MAX_M, prefill above).
 * Other arguments, checks and errors as gptq_w4a16_gemm, plus
 * GPTQ_ERR_NULL for a NULL qzeros, GPTQ_ERR_SHAPE for N % 32 != 0, and
 * GPTQ_ERR_ALIAS when y overlaps qzeros.
 */
GPTQ_API int gptq_w4a16_gemm_asym(const uint16_t* x, const int32_t* qweight,
                                  const uint16_t* scales, const int32_t* qzeros, int64_t M,
                                  int64_t K, int64_t N, int32_t group, uint16_t* y,
                                  void* stream);

/*
 * The layer with a LoRA adapter on its path:
 *   T = fp16(X . lora_a^T)                       [M, rank]
 *   Y = fp16(X . dequant(qweight, scales) + T . lora_b^T)
 * The GPTQ-Pro README ("Runtime contract") puts LoRA adapters on the linear
 * path; the GPTQModel README ("PEFT LoRA Training and Adapter Loading") keeps
 * the adapter separate from the packed weights.  Read with PEFT's layouts:
 *   lora_a   [rank, K] FP16 bits, device (lora_A.weight)
 *   lora_b   [N, rank] FP16 bits, device (lora_B.weight), with the adapter's
 *            scaling (alpha / rank) already multiplied in
 *   rank     16 .. GPTQ_MAX_LORA_RANK, a multiple of 16
 *   t_work   [M, rank] FP16 bits, device, caller-owned: receives T (the
 *            adapter's down-projection, rounded to FP16 like the adapter's
 *            own output); must not overlap any other argument
 * T is summed in FP32 and rounded to FP16; T . lora_b^T is added to the
 * layer's FP32 accumulator (the adapter's rank is extra K of the same
 * tensor-core product) and Y is rounded once.  Up to GPTQ_LORA_DECODE_MAX_M
 * tokens the layer runs on the decode kernel, and when its column blocks
 * leave SMs free T is computed by CTAs of that same launch, on those SMs,
 * and handed over through a counter in the library's static device memory
 * (one of 1024 slots, taken in turn by successive calls on the device; the
 * last reader clears it): one launch.  Otherwise two launches on `stream`: T,
 * then the layer (decode kernel, or the prefill kernel above
 * GPTQ_LORA_DECODE_MAX_M tokens), which may start while T is computed and
 * waits for T only before reading it.  Calls that may run at the same time
 * on different streams take different slots; a CUDA graph that holds such a
 * call keeps its slot, so one graph must not be replayed on two streams at
 * once.  Other arguments, checks
 * and errors as gptq_w4a16_gemm, plus GPTQ_ERR_NULL for a NULL lora_a, lora_b
 * or t_work (when M > 0), GPTQ_ERR_SHAPE for a rank out of range, and
 * GPTQ_ERR_ALIAS when t_work or y overlaps any other buffer.
 */
GPTQ_API int gptq_w4a16_gemm_lora(const uint16_t* x, const int32_t* qweight,
                                  const uint16_t* scales, int64_t M, int64_t K, int64_t N,
                                  int32_t group, const uint16_t* lora_a,
                                  const uint16_t* lora_b, int64_t rank, uint16_t* t_work,
                                  uint16_t* y, void* stream);

/*
 * gptq_w4a16_gemm_lora without a caller-provided T buffer.  The pages have no
 * counterpart of this entry point: it exists for callers that cannot hand
 * the library device scratch.  T [M, rank] is kept in one fixed device buffer
 * inside the library (GPTQ_LORA_SCRATCH_BYTES per device, part of the
 * library's static device memory), so the call allocates nothing.
 *   M * rank * 2 must not exceed GPTQ_LORA_SCRATCH_BYTES, else GPTQ_ERR_SHAPE
 *   (checked before anything is enqueued).
 * T is written in full before it is read, so nothing in the buffer has to
 * start at zero.  Every call on a device uses the same buffer: two calls
 * whose executions may overlap (streams without an ordering between them, or
 * host threads enqueueing concurrently on different streams) race on it and
 * can return wrong results; calls ordered on one stream are safe.  Results
 * are bit-identical to gptq_w4a16_gemm_lora.  Other arguments, checks and
 * errors as gptq_w4a16_gemm_lora (without t_work).
 */
GPTQ_API int gptq_w4a16_gemm_lora_noalloc(const uint16_t* x, const int32_t* qweight,
                                          const uint16_t* scales, int64_t M, int64_t K,
                                          int64_t N, int32_t group, const uint16_t* lora_a,
                                          const uint16_t* lora_b, int64_t rank, uint16_t* y,
                                          void* stream);

/*
 * The layer with act-order weights (GPTQ's desc_act=True checkpoints), whose
 * input channels each carry their own group index:
 *   Y = X . W,  W[k,n] = fp16((q[k,n] - 8) * scales[g_idx[k], n])
 * The GPTQ-Pro README ("Runtime contract") runs desc_act=False only and puts
 * act order outside its contract; the GPTQModel wiki names desc_act as
 * activation ordering.  Neither gives its storage; read as GPTQ's:
 *   g_idx    [K] int32, device, 16-byte aligned, 0 <= g_idx[k] < n_groups;
 *            any assignment of channels to groups (group sizes need not be
 *            equal); qweight keeps the channels in their own order
 *   scales   [n_groups, N] FP16 bits, device
 *   n_groups 1 .. GPTQ_GIDX_MAX_GROUPS (each CTA keeps the scale rows of its
 *            128 columns in shared memory)
 * With g_idx[k] = floor(k / G) the layer is gptq_w4a16_gemm's with group G,
 * and for M <= GPTQ_DECODE_MAX_M the result is the same bit for bit.  Runs on
 * the decode kernel for every M (tiles of at most 64 tokens; above that the
 * weights are streamed once per tile).  An index out of range is clamped
 * into 0 .. n_groups-1 for reading (no access outside scales) and reported
 * as GPTQ_ERR_INDEX by gptq_device_error; the output is then undefined.
 * Other arguments, checks and errors as gptq_w4a16_gemm (no group argument),
 * plus GPTQ_ERR_NULL for a NULL g_idx, GPTQ_ERR_SHAPE for n_groups out of
 * range, and GPTQ_ERR_ALIAS when y overlaps g_idx.
 */
GPTQ_API int gptq_w4a16_gemm_gidx(const uint16_t* x, const int32_t* qweight,
                                  const uint16_t* scales, const int32_t* g_idx, int64_t M,
                                  int64_t K, int64_t N, int64_t n_groups, uint16_t* y,
                                  void* stream);

/*
 * W[K, N] = dequant(qweight, scales) as FP16 bits, each value rounded once from
 * the exact (q - 8) * s (a debugging and verification entry; the GEMM never
 * materialises W).  w_out must not overlap qweight or scales.
 */
GPTQ_API int gptq_dequant(const int32_t* qweight, const uint16_t* scales, int64_t K, int64_t N,
                 int32_t group, uint16_t* w_out, void* stream);

/*
 * The dispatcher, observable: which kernel gptq_w4a16_gemm would launch for
 * this shape and with how many K-splits (1 when the kernel does not split K).
 * Validates the shape and group like the GEMM (not the pointers); needs a
 * current CUDA device of compute capability 10.0 (the split depends on its SM
 * count).  Either output pointer may be NULL.
 */
GPTQ_API int gptq_w4a16_select(int64_t M, int64_t K, int64_t N, int32_t group,
                      int32_t* kernel_id, int32_t* split_k);

/* Static, human-readable name of a gptq_status value. */
GPTQ_API const char* gptq_status_string(int status);

/*
 * Reads and clears the device-side error word of the current device: 0 when
 * no kernel gave up a bounded wait or met a bad index since the last call,
 * else GPTQ_ERR_TIMEOUT or GPTQ_ERR_INDEX.  Synchronises the current device.
 * Kernels never trap: a wait that exceeds its bound records the error here,
 * abandons the output tile and exits.  After an error it also clears the
 * library's adapter hand-over counters (static device memory), which a kernel
 * that gave up may have left set.
 */
GPTQ_API int gptq_device_error(void);

/* Library version as "major.minor.patch". */
GPTQ_API const char* gptq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_W4A16_H */
