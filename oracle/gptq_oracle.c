/*
 * CPU oracle for the symmetric INT4 GPTQ W4A16 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or table with the CUDA
 * library.
 *
 * What it computes (GPTQ-Pro README, "Runtime contract": symmetric GPTQ INT4,
 * FP16 activations, desc_act=False, native int32 qweight, group sizes
 * -1/16/32/64/128/256/512/1024; GPTQModel wiki "Installation and Quickstart",
 * "Defaults and compatibility decisions": sym True, pack_dtype torch.int32):
 *
 *   code   q[k,n] = (uint32(qweight[k/8, n]) >> (4*(k%8))) & 0xF
 *   group  g(k)   = floor(k / G)         (G = K when group == -1)
 *   weight W[k,n] = fp16_RNE((q[k,n] - 8) * scales[g(k), n])
 *   output Y[m,n] = sum_k x[m,k] * W[k,n]   in binary64, k ascending
 *
 * The pages fix none of: the nibble order inside a word, how a group that
 * does not divide K ends, or where rounding happens.  The readings used are:
 * lowest nibble = lowest k; the last group is ragged (n_groups = ceil(K/G));
 * the product (q-8)*s is formed exactly and rounded once to binary16 with
 * round-to-nearest-even.  Parity is pinned by the tests (exhaustive binary16
 * rounding, closed forms, brute force on tiny shapes, round trips).
 *
 * Every routine here is deliberately plain: one element at a time, no
 * blocking, no vectorisation; OpenMP threads only split independent outputs.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads split the independent outputs (columns or listed entries) only;
 * every output's sum over k is still formed by one thread in ascending k, so
 * the result does not depend on the thread count. */
void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---- IEEE 754-2008 binary16: 1 sign bit, 5 exponent bits (bias 15),
 *      10 fraction bits.  emin = -14, precision p = 11. ---------------------- */

double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int exp = (h >> 10) & 0x1F;
    int frac = h & 0x3FF;
    double v;
    if (exp == 0x1F) {
        v = frac ? NAN : INFINITY;
    } else if (exp == 0) {
        v = ldexp((double)frac, -24);            /* subnormal: frac * 2^-24 */
    } else {
        v = ldexp((double)(1024 + frac), exp - 25); /* (1.frac) * 2^(exp-15) */
    }
    return sign ? -v : v;
}

/* Round a binary64 value to the nearest binary16 value, ties to even.
 * Values at or beyond the overflow threshold (65520) become infinity. */
uint16_t oracle_double_to_half(double v)
{
    if (isnan(v)) return 0x7E00;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7C00;

    /* a lies in [2^E, 2^(E+1)); binary16 spacing there is 2^(E-10), and in
     * the subnormal range (E < -14) it is the fixed 2^-24. */
    int e2;
    frexp(a, &e2);                 /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;
    if (E < -14) E = -14;
    double ulp = ldexp(1.0, E - 10);
    double units = a / ulp;        /* exact: division by a power of two */
    double lower = floor(units);
    double rem = units - lower;    /* exact */
    double n;
    if (rem > 0.5) n = lower + 1.0;
    else if (rem < 0.5) n = lower;
    else n = (fmod(lower, 2.0) == 0.0) ? lower : lower + 1.0;  /* tie: even */

    double r = n * ulp;            /* the rounded magnitude */
    if (r >= 65536.0) return sign | 0x7C00;   /* beyond 65504: infinity */
    if (r < ldexp(1.0, -14)) {
        /* subnormal (or the smallest normal reached by rounding up) */
        uint32_t m = (uint32_t)(r / ldexp(1.0, -24));
        return sign | (uint16_t)m;  /* m == 1024 encodes 2^-14 correctly */
    }
    int re2;
    frexp(r, &re2);
    int RE = re2 - 1;              /* r in [2^RE, 2^(RE+1)) */
    uint32_t mant = (uint32_t)(r / ldexp(1.0, RE - 10)) - 1024u;
    return sign | (uint16_t)(((RE + 15) << 10) | mant);
}

void oracle_round_to_half(const double* v, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_double_to_half(v[i]);
}

/* ---- packing ----------------------------------------------------------- */

/* code of row k, column n from qweight [K/8, N] */
static int code_at(const int32_t* qweight, int64_t N, int64_t k, int64_t n)
{
    uint32_t word = (uint32_t)qweight[(k / 8) * N + n];
    return (int)((word >> (4 * (k % 8))) & 0xFu);
}

void oracle_unpack(const int32_t* qweight, int64_t K, int64_t N, uint8_t* codes)
{
    for (int64_t k = 0; k < K; ++k)
        for (int64_t n = 0; n < N; ++n)
            codes[k * N + n] = (uint8_t)code_at(qweight, N, k, n);
}

void oracle_pack(const uint8_t* codes, int64_t K, int64_t N, int32_t* qweight)
{
    for (int64_t i = 0; i < K / 8; ++i)
        for (int64_t n = 0; n < N; ++n) {
            uint32_t word = 0;
            for (int j = 0; j < 8; ++j)
                word |= ((uint32_t)(codes[(8 * i + j) * N + n] & 0xF)) << (4 * j);
            qweight[i * N + n] = (int32_t)word;
        }
}

/* ---- groups ------------------------------------------------------------ */

int64_t oracle_num_groups(int64_t K, int32_t group)
{
    if (group == -1 || group >= K) return 1;
    return (K + group - 1) / group;
}

static int64_t group_of(int64_t k, int32_t group)
{
    return group == -1 ? 0 : k / group;
}

/* ---- dequantisation ---------------------------------------------------- */

static uint16_t dequant_at(const int32_t* qweight, const uint16_t* scales,
                           int64_t N, int32_t group, int64_t k, int64_t n)
{
    double q = (double)code_at(qweight, N, k, n);
    double s = oracle_half_to_double(scales[group_of(k, group) * N + n]);
    return oracle_double_to_half((q - 8.0) * s);   /* exact product, one rounding */
}

void oracle_dequant(const int32_t* qweight, const uint16_t* scales, int64_t K,
                    int64_t N, int32_t group, uint16_t* w)
{
    #pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < K; ++k)
        for (int64_t n = 0; n < N; ++n)
            w[k * N + n] = dequant_at(qweight, scales, N, group, k, n);
}

/* ---- the layer --------------------------------------------------------- */

/* Y[m,n] for every (m, n); y is binary64 [M, N]. */
int oracle_gemm(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                int64_t M, int64_t K, int64_t N, int32_t group, double* y)
{
    uint16_t* w = (uint16_t*)malloc((size_t)(K * N) * sizeof(uint16_t));
    if (!w) return 1;
    oracle_dequant(qweight, scales, K, N, group, w);
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += oracle_half_to_double(x[m * K + k]) * oracle_half_to_double(w[k * N + n]);
            y[m * N + n] = acc;
        }
    free(w);
    return 0;
}

/* Y[ms[i], ns[i]] for a list of entries (for problems too large to compute
 * whole); each entry dequantises its own column on the fly. */
void oracle_gemm_entries(const uint16_t* x, const int32_t* qweight,
                         const uint16_t* scales, int64_t M, int64_t K, int64_t N,
                         int32_t group, int64_t count, const int64_t* ms,
                         const int64_t* ns, double* out)
{
    (void)M;
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = ms[i], n = ns[i];
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k)
            acc += oracle_half_to_double(x[m * K + k])
                 * oracle_half_to_double(dequant_at(qweight, scales, N, group, k, n));
        out[i] = acc;
    }
}

/* Y rows ms[0..count) in full: out is binary64 [count, N].  Column n's
 * weights are dequantised once and used for every listed row. */
void oracle_gemm_rows(const uint16_t* x, const int32_t* qweight,
                      const uint16_t* scales, int64_t M, int64_t K, int64_t N,
                      int32_t group, int64_t count, const int64_t* ms, double* out)
{
    (void)M;
    #pragma omp parallel for schedule(dynamic, 64)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t i = 0; i < count; ++i) out[i * N + n] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double w = oracle_half_to_double(dequant_at(qweight, scales, N, group, k, n));
            for (int64_t i = 0; i < count; ++i)
                out[i * N + n] += oracle_half_to_double(x[ms[i] * K + k]) * w;
        }
    }
}

/* ---- LoRA adapter on the linear path ------------------------------------
 *
 * GPTQ-Pro README, "Runtime contract" (adapters: LoRA on the GPTQ-Pro linear
 * path) and GPTQModel README, "PEFT LoRA Training and Adapter Loading" (the
 * adapter stays separate from the packed weights).  Read as the usual LoRA
 * delta with PEFT's layouts and the adapter's scaling already in lora_b:
 *     T[m,j] = fp16_RNE( sum_k x[m,k] * lora_a[j,k] )      lora_a [r, K]
 *     Y[m,n] = sum_k x[m,k] * W[k,n] + sum_j T[m,j] * lora_b[n,j]   lora_b [N, r]
 * T is rounded to FP16 (the adapter's dtype); Y is the binary64 sum.
 */

/* t (FP16 bits) [M, r] = fp16(x . lora_a^T), binary64 sums, k ascending. */
void oracle_lora_down(const uint16_t* x, const uint16_t* lora_a, int64_t M, int64_t K,
                      int64_t r, uint16_t* t)
{
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += oracle_half_to_double(x[m * K + k]) * oracle_half_to_double(lora_a[j * K + k]);
            t[m * r + j] = oracle_double_to_half(acc);
        }
}

/* y [count, N] (binary64) += t[ms[i], :] . lora_b^T, j ascending. */
void oracle_lora_up_add(const uint16_t* t, const uint16_t* lora_b, int64_t r, int64_t N,
                        int64_t count, const int64_t* ms, double* y)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t j = 0; j < r; ++j)
                acc += oracle_half_to_double(t[ms[i] * r + j]) * oracle_half_to_double(lora_b[n * r + j]);
            y[i * N + n] += acc;
        }
}

/* ---- asymmetric zero points ----------------------------------------------
 *
 * GPTQModel wiki "Installation and Quickstart", "Defaults and compatibility
 * decisions" (sym is True by default, and not every backend accepts
 * asymmetric weights) and GPTQ-Pro README, "Runtime contract" (asymmetric
 * weights lie outside that fork's contract).  Read with GPTQ's packed
 * zero points, eight 4-bit codes per int32 along N (lowest nibble = lowest
 * n, as the weights along K), each taken as stored:
 *     z[g,n] = (uint32(qzeros[g, n/8]) >> 4*(n%8)) & 0xF   qzeros [n_groups, N/8]
 *     W[k,n] = fp16_RNE((q[k,n] - z[g(k),n]) * scales[g(k),n])
 * With every z = 8 this is the symmetric layer above.
 */

static int zero_at(const int32_t* qzeros, int64_t N, int64_t g, int64_t n)
{
    uint32_t word = (uint32_t)qzeros[g * (N / 8) + n / 8];
    return (int)((word >> (4 * (n % 8))) & 0xFu);
}

static uint16_t dequant_asym_at(const int32_t* qweight, const uint16_t* scales,
                                const int32_t* qzeros, int64_t N, int32_t group, int64_t k,
                                int64_t n)
{
    int64_t g = group_of(k, group);
    double q = (double)code_at(qweight, N, k, n);
    double z = (double)zero_at(qzeros, N, g, n);
    double s = oracle_half_to_double(scales[g * N + n]);
    return oracle_double_to_half((q - z) * s);   /* exact product, one rounding */
}

void oracle_dequant_asym(const int32_t* qweight, const uint16_t* scales, const int32_t* qzeros,
                         int64_t K, int64_t N, int32_t group, uint16_t* w)
{
    #pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < K; ++k)
        for (int64_t n = 0; n < N; ++n)
            w[k * N + n] = dequant_asym_at(qweight, scales, qzeros, N, group, k, n);
}

/* Y rows ms[0..count) of the asymmetric layer, binary64 [count, N]. */
void oracle_gemm_asym_rows(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                           const int32_t* qzeros, int64_t M, int64_t K, int64_t N,
                           int32_t group, int64_t count, const int64_t* ms, double* out)
{
    (void)M;
    #pragma omp parallel for schedule(dynamic, 64)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t i = 0; i < count; ++i) out[i * N + n] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double w = oracle_half_to_double(
                dequant_asym_at(qweight, scales, qzeros, N, group, k, n));
            for (int64_t i = 0; i < count; ++i)
                out[i * N + n] += oracle_half_to_double(x[ms[i] * K + k]) * w;
        }
    }
}

/* ---- act-order weights (per-channel group index) -------------------------
 *
 * GPTQ-Pro README, "Runtime contract" (desc_act=False only; act-order
 * checkpoints lie outside that fork's contract) and GPTQModel wiki
 * "Installation and Quickstart", "Defaults and compatibility decisions"
 * (desc_act is activation ordering).  With act order the quantiser visits the
 * input channels in a permuted order, so a group is no longer a run of
 * consecutive k.  The pages give no storage for it; read with GPTQ's group
 * index per input channel, qweight keeping the channels in their own order:
 *     g_idx [K] int32,  0 <= g_idx[k] < n_groups
 *     W[k,n] = fp16_RNE((q[k,n] - 8) * scales[g_idx[k], n])
 * With g_idx[k] = floor(k / G) this is the layer above.
 */

static int gidx_valid(const int32_t* g_idx, int64_t K, int64_t n_groups)
{
    for (int64_t k = 0; k < K; ++k)
        if (g_idx[k] < 0 || g_idx[k] >= n_groups) return 0;
    return 1;
}

static uint16_t dequant_gidx_at(const int32_t* qweight, const uint16_t* scales,
                                const int32_t* g_idx, int64_t N, int64_t k, int64_t n)
{
    double q = (double)code_at(qweight, N, k, n);
    double s = oracle_half_to_double(scales[(int64_t)g_idx[k] * N + n]);
    return oracle_double_to_half((q - 8.0) * s);   /* exact product, one rounding */
}

/* W (FP16 bits) [K, N]; returns 1, writing nothing, if an index is out of range. */
int oracle_dequant_gidx(const int32_t* qweight, const uint16_t* scales, const int32_t* g_idx,
                        int64_t K, int64_t N, int64_t n_groups, uint16_t* w)
{
    if (!gidx_valid(g_idx, K, n_groups)) return 1;
    #pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < K; ++k)
        for (int64_t n = 0; n < N; ++n)
            w[k * N + n] = dequant_gidx_at(qweight, scales, g_idx, N, k, n);
    return 0;
}

/* Y rows ms[0..count) of the act-order layer, binary64 [count, N], k
 * ascending; returns 1, writing nothing, if an index is out of range. */
int oracle_gemm_gidx_rows(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                          const int32_t* g_idx, int64_t M, int64_t K, int64_t N,
                          int64_t n_groups, int64_t count, const int64_t* ms, double* out)
{
    (void)M;
    if (!gidx_valid(g_idx, K, n_groups)) return 1;
    #pragma omp parallel for schedule(dynamic, 64)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t i = 0; i < count; ++i) out[i * N + n] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double w = oracle_half_to_double(dequant_gidx_at(qweight, scales, g_idx, N, k, n));
            for (int64_t i = 0; i < count; ++i)
                out[i * N + n] += oracle_half_to_double(x[ms[i] * K + k]) * w;
        }
    }
    return 0;
}
