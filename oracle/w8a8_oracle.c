/*
 * w8a8_oracle.c -- plain, slow, obviously correct CPU definition of the W8A8
 * int8-dynamic linear layer.  TEST INFRASTRUCTURE ONLY: the tests, the smoke
 * check and the benchmark's CPU-baseline leg call it; the product path never
 * does.  It shares no source with the CUDA library.
 *
 * What it computes, and where that is stated:
 *
 *  - Scheme: int8 weights with one fp32 scale per output channel, and dynamic
 *    per-token symmetric int8 activations ("Issue 5 probe: int8 quantized DiT
 *    serve paths on the RTX 3090 (24 GB)", section "Round two ... W8A8
 *    int8-dynamic", first paragraph and the artifact note on fp32 per-channel
 *    scales; "Qwen-Image-2.1: TE AutoRound-AWQ on GPU + all-resident
 *    single-3090 stack", section "Whole-pipeline follow-up", on TorchAO's
 *    per-token activation and per-channel weight quantization).  Activation
 *    scales are computed online at every call; static scales are not part of
 *    the method ("Int8 Quantization" user guide, "Overview" and the
 *    "Parameters" table, activation_scheme = "dynamic").
 *
 *  - The pages name the scheme but print no formula.  The formula used here is
 *    the plain symmetric one:  s = max_k |x[k]| / 127  (fp32, IEEE division,
 *    round to nearest even),  q[k] = clamp(rint(x[k] / s), -127, 127)  with
 *    rint rounding half to even.  A row with max |x| == 0 has s = 0 and q = 0.
 *    The same rule applied to a weight row gives s_w and Wq.
 *
 *  - The GEMM is exact integer arithmetic: acc[m][n] = sum_k q[m][k]*Wq[n][k]
 *    (summed in int64 here and checked to fit int32).
 *
 *  - The epilogue applies both scales and the bias in fp32, one rounded IEEE
 *    operation at a time, in this order:
 *        y32 = ((float)acc * s_a[m]) * s_w[n];   y32 = y32 + (float)bias[n];
 *    then rounds y32 to bf16 (nearest, ties to even).  The "Round two" section
 *    records that dropping the x s_a factor is the mistake that made a probe's
 *    output/reference norm ratio equal the mean activation scale.
 *
 * Build: plain C99, -O2 -fno-fast-math -ffp-contract=off, no flush-to-zero,
 * OpenMP over rows (see build.py next to this file).  On x86-64 float
 * arithmetic is SSE single precision, so each operation above is one IEEE
 * binary32 operation in round-to-nearest-even.
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- bf16 <-> fp32 ------------------------------------------------------ */

/* bf16 is the top 16 bits of an IEEE binary32: widening is exact. */
static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Narrow a finite float to bf16 bits, rounding to nearest, ties to even:
 * add half of the dropped range (minus one when the kept LSB is 0) and
 * truncate.  NaN keeps a quiet NaN; +-inf passes through. */
static uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u) {
        if (u & 0x007fffffu) return (uint16_t)((u >> 16) | 0x0040u);
        return (uint16_t)(u >> 16);
    }
    uint32_t keep_lsb = (u >> 16) & 1u;
    u += 0x7fffu + keep_lsb;
    return (uint16_t)(u >> 16);
}

/* ---- per-row symmetric quantization -------------------------------------- */

/* One row: s = amax/127, q = clamp(rint(v/s), -127, 127). */
static void quant_one_row(const uint16_t *xr, int64_t cols, int8_t *qr, float *s_out)
{
    float amax = 0.0f;
    for (int64_t c = 0; c < cols; ++c) {
        float a = fabsf(bf16_to_f32(xr[c]));
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        *s_out = 0.0f;
        for (int64_t c = 0; c < cols; ++c) qr[c] = 0;
        return;
    }
    float s = amax / 127.0f;
    *s_out = s;
    for (int64_t c = 0; c < cols; ++c) {
        float t = bf16_to_f32(xr[c]) / s;  /* IEEE binary32 division */
        float r = nearbyintf(t);           /* current mode: nearest, ties even */
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        qr[c] = (int8_t)r;
    }
}

/* Quantize `rows` rows of bf16 bits x (row stride ldx elements) into int8 q
 * (row stride ldq) and fp32 scales s.  Returns 0, or -1 on bad arguments. */
int w8a8_oracle_quant_rows(const uint16_t *x, int64_t rows, int64_t cols, int64_t ldx,
                           int8_t *q, int64_t ldq, float *s)
{
    if (!x || !q || !s || rows < 0 || cols < 0 || ldx < cols || ldq < cols) return -1;
    if (fegetround() != FE_TONEAREST) fesetround(FE_TONEAREST);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
#ifdef _OPENMP
        if (fegetround() != FE_TONEAREST) fesetround(FE_TONEAREST);
#endif
        quant_one_row(x + r * ldx, cols, q + r * ldq, s + r);
    }
    return 0;
}

/* ---- exact integer GEMM -------------------------------------------------- */

/* acc[m*ldacc + n] = sum_k a[m*lda + k] * b[n*ldb + k], exact.  The sums are
 * formed in int64; the function returns the number of outputs that do not fit
 * int32 (those are stored truncated and must be treated as a failure). */
int64_t w8a8_oracle_gemm_i32(const int8_t *a, int64_t M, int64_t lda,
                             const int8_t *b, int64_t N, int64_t ldb, int64_t K,
                             int32_t *acc, int64_t ldacc)
{
    if (!a || !b || !acc || M < 0 || N < 0 || K < 0) return -1;
    int64_t overflow = 0;
#pragma omp parallel for schedule(static) reduction(+ : overflow)
    for (int64_t m = 0; m < M; ++m) {
        const int8_t *ar = a + m * lda;
        for (int64_t n = 0; n < N; ++n) {
            const int8_t *br = b + n * ldb;
            int64_t sum = 0;
            for (int64_t k = 0; k < K; ++k) sum += (int64_t)ar[k] * (int64_t)br[k];
            if (sum > INT32_MAX || sum < INT32_MIN) overflow += 1;
            acc[m * ldacc + n] = (int32_t)sum;
        }
    }
    return overflow;
}

/* ---- fp32 epilogue -------------------------------------------------------- */

/* y32 = ((float)acc * s_a[m]) * s_w[n] (+ (float)bias[n]); y = bf16_rne(y32).
 * bias may be NULL; y32 or y may be NULL when not wanted. */
int w8a8_oracle_epilogue(const int32_t *acc, int64_t M, int64_t N, int64_t ldacc,
                         const float *s_a, const float *s_w, const uint16_t *bias,
                         float *y32, int64_t ldy32, uint16_t *y, int64_t ldy)
{
    if (!acc || !s_a || !s_w || M < 0 || N < 0) return -1;
    if (fegetround() != FE_TONEAREST) fesetround(FE_TONEAREST);
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            float v = (float)acc[m * ldacc + n];  /* int32 -> binary32, nearest */
            v = v * s_a[m];
            v = v * s_w[n];
            if (bias) v = v + bf16_to_f32(bias[n]);
            if (y32) y32[m * ldy32 + n] = v;
            if (y) y[m * ldy + n] = f32_to_bf16_rne(v);
        }
    }
    return 0;
}

/* ---- whole layer ---------------------------------------------------------- */

/* The full definition for M rows of x against pre-quantized weights.  q_out,
 * s_a_out, acc_out, y32_out are caller buffers ([M,K], [M], [M,N], [M,N],
 * dense); y_out is [M,N] bf16 bits, dense.  Returns the int32-overflow count
 * (0 expected), or -1 on bad arguments. */
int64_t w8a8_oracle_linear(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                           const int8_t *wq, const float *s_w, const uint16_t *bias, int64_t N,
                           int8_t *q_out, float *s_a_out, int32_t *acc_out,
                           float *y32_out, uint16_t *y_out)
{
    if (w8a8_oracle_quant_rows(x, M, K, ldx, q_out, K, s_a_out) != 0) return -1;
    int64_t ov = w8a8_oracle_gemm_i32(q_out, M, K, wq, N, K, K, acc_out, N);
    if (ov < 0) return -1;
    if (w8a8_oracle_epilogue(acc_out, M, N, N, s_a_out, s_w, bias, y32_out, N, y_out, N) != 0)
        return -1;
    return ov;
}

/* ---- W8A16: int8 weights, bf16 activations ------------------------------- */

/*
 * The weight-only variant the pages ran first ("Issue 5 probe: int8 quantized
 * DiT serve paths on the RTX 3090 (24 GB)", section "Round one: int8
 * weight-only via compressed-tensors": int8 weight-only (W8A16),
 * per-output-channel symmetric; the activations stay bf16).  With one scale
 * per output channel the dequantized product factors as
 *     y[m][n] = s_w[n] * sum_k x[m][k] * q[n][k] + bias[n].
 * Each product x * q is exact in binary32 (an 8-bit significand times a
 * 7-bit integer), so the only rounding inside the sum is the summation
 * itself, whose order a tensor core leaves open.  The oracle forms the sum in
 * binary64 (exact whenever the products span fewer than about 53 - 15 -
 * log2 K binades, as for the tests' inputs; in general within K * 2^-53 of
 * the exact sum, relative to sum |x * q|), rounds it once to binary32
 * (acc32), then applies the scale and the bias as separately rounded
 * binary32 operations and rounds to bf16:
 *     y32 = acc32 * s_w[n] (+ (float)bias[n]),  y = bf16(y32).
 * abs_sum[m][n] = sum_k |x * q| (binary64, rounded to binary32) bounds how
 * far any binary32 summation order can drift from the exact sum:
 * |sum_fp32 - sum| <= gamma_K * abs_sum,  gamma_K = K u / (1 - K u),
 * u = 2^-24 (the standard bound for recursive summation in any order).
 */
int w8a16_oracle_linear(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                        const int8_t *wq, const float *s_w, const uint16_t *bias, int64_t N,
                        float *acc32_out, float *abs_sum_out, float *y32_out, uint16_t *y_out)
{
    if (!x || !wq || !s_w || M < 0 || N < 0 || K < 0 || ldx < K) return -1;
    if (fegetround() != FE_TONEAREST) fesetround(FE_TONEAREST);
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double sum = 0.0, asum = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = (double)bf16_to_f32(x[m * ldx + k]) * (double)wq[n * K + k];
                sum += p;
                asum += fabs(p);
            }
            float acc = (float)sum;
            float v = acc * s_w[n];
            if (bias) v = v + bf16_to_f32(bias[n]);
            if (acc32_out) acc32_out[m * N + n] = acc;
            if (abs_sum_out) abs_sum_out[m * N + n] = (float)asum;
            if (y32_out) y32_out[m * N + n] = v;
            if (y_out) y_out[m * N + n] = f32_to_bf16_rne(v);
        }
    }
    return 0;
}

/* ---- packed int32 weight storage ----------------------------------------- */

/*
 * The serialized form of an int8 weight: each code stored as an unsigned byte
 * biased by 128, four bytes per int32 word ("Issue 5 probe: int8 quantized
 * DiT serve paths on the RTX 3090 (24 GB)", section "Artifact (outside Git,
 * under the helper state root)": the quantized transformer is built with
 * compressed-tensors' pack_to_int32).  The
 * pages fix the bias and the four-per-word ratio; the order inside a word is
 * taken as consecutive codes along K, the first in the least significant
 * byte.  packed is int32 [N][K/4] (K a multiple of 4), Wq int8 [N][K].
 */
void w8a8_oracle_pack_int32(const int8_t *wq, int64_t N, int64_t K, int32_t *packed)
{
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < K / 4; ++g) {
            uint32_t word = 0;
            for (int j = 0; j < 4; ++j) {
                uint32_t biased = (uint32_t)((int32_t)wq[n * K + 4 * g + j] + 128);
                word |= biased << (8 * j);
            }
            packed[n * (K / 4) + g] = (int32_t)word;
        }
    }
}

void w8a8_oracle_unpack_int32(const int32_t *packed, int64_t N, int64_t K, int8_t *wq)
{
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            uint32_t word = (uint32_t)packed[n * (K / 4) + k / 4];
            int32_t biased = (int32_t)((word >> (8 * (k % 4))) & 0xFFu);
            wq[n * K + k] = (int8_t)(biased - 128);
        }
    }
}

/* ---- helpers for the Python side ---------------------------------------- */

uint16_t w8a8_oracle_f32_to_bf16(float f) { return f32_to_bf16_rne(f); }

void w8a8_oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int w8a8_oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
