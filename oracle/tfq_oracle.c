/*
 * tfq_oracle.c -- plain, slow, obviously-correct CPU oracle for the W8A8
 * scaled-FP8 Linear.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline / reference arm may load this library.  The
 * product path (the CUDA library and its Python binding) never calls it and
 * shares no code, header, table or constant with it.
 *
 * What it computes, and where the pages define it:
 *
 *  - Symmetric absmax quantization with one scale per row
 *      s = max|x| / qmax,   q = cast(clamp(x / s, -qmax, qmax))
 *    TeleFuser "Quantization" page, section "Scaled FP8 checkpoints: W8A8"
 *    (per-row scaled-FP8 formula); qmax = max(E4M3FN) = 448 there, and the
 *    reduced qmax values 14 and 7 come from the LightX2V "模型量化技术" page,
 *    section "MiniMax-H3 FP8 FP16 累加" (scale = max(abs(x)) / qmax per row).
 *  - The INT8 variant  s = max|x| / 127,  q = clamp(round(x / s), -128, 127)
 *    TeleFuser "Quantization" page, section "Core ideas" (integer formula),
 *    one scale per output row as in section "Offline conversion".
 *  - MXFP8 (32-value blocks, E8M0 power-of-two scales) and its block-scaled
 *    GEMM: TeleFuser "Quantization" page, section "Offline conversion" names
 *    the format; the conversion is the OCP MX v1.0 one (see below).
 *  - The scaled GEMM  y[m,n] = s_a[m] s_w[n] sum_k q_a[m,k] q_w[n,k] (+ b[n])
 *    TeleFuser "Quantization" page, sections "Scaled FP8 checkpoints" and
 *    "tf-kernel FP8: online W8A8" (per-token activations, per-output-channel
 *    weights, scaled GEMM with BF16 output).
 *
 * Readings taken where the pages are silent (each one is listed with its
 * reason in the design notes of the repository):
 *  - arithmetic: the bf16 input is widened to fp32 exactly; the scale and
 *    the quotient x/s are single IEEE fp32 divisions, round-to-nearest-even;
 *  - an all-zero (or tiny) row uses amax = max(amax, 1e-12f);
 *  - the FP8 "cast" is round-to-nearest-even onto the E4M3FN grid,
 *    saturating at +-448, sign kept (so -0 and negative underflow give 0x80);
 *  - INT8 "round" is round-half-to-even;
 *  - the GEMM accumulates products of decoded codes in double (exact for the
 *    sizes in use: every product of two E4M3 values is a multiple of 2^-18
 *    below 2^18, so partial sums stay exact in 53 bits for K < 2^17), then
 *    applies the scales and the bias in double; no rounding to bf16 is done
 *    here: the comparison with a bf16 result happens in the tests.
 *
 * Compile with IEEE semantics: no -ffast-math, -ffp-contract=off, and SSE
 * arithmetic (x86-64 evaluates float in float, FLT_EVAL_METHOD == 0).
 */
#include <float.h>
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#if defined(FLT_EVAL_METHOD) && FLT_EVAL_METHOD != 0
#error "the oracle needs float arithmetic evaluated in float"
#endif

/* ------------------------------------------------------------------ */
/* bf16 -> fp32 widening: a bf16 value is the upper half of an fp32.   */
/* ------------------------------------------------------------------ */
static float bf16_bits_to_float(uint16_t bits)
{
    uint32_t w = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return f;
}

/* ------------------------------------------------------------------ */
/* E4M3FN, from the OCP 8-bit floating point format definition:        */
/*   1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits;            */
/*   exponent field 0 holds subnormals m * 2^-9;                       */
/*   otherwise (8 + m) * 2^(e - 10);                                   */
/*   S.1111.111 is NaN, there is no infinity, the largest finite       */
/*   magnitude is 1.75 * 2^8 = 448 (code 0x7E).                        */
/* ------------------------------------------------------------------ */
double tfq_oracle_e4m3_decode(uint8_t code)
{
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);
    else
        mag = ldexp((double)(8 + m), e - 10);
    return sign ? -mag : mag;
}

/* Round a non-negative double to an integer, ties to the even integer. */
static double round_half_even_nonneg(double v)
{
    double f = floor(v);
    double frac = v - f; /* exact: v and f share the binade or f is 0 */
    if (frac > 0.5)
        return f + 1.0;
    if (frac < 0.5)
        return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/*
 * Encode an fp32 value to the nearest E4M3FN code, ties to even mantissa,
 * saturating at +-448.  Every E4M3FN magnitude with exponent e (e >= -6;
 * subnormals share the e = -6 spacing) is a multiple of 2^(e-3), so the
 * value is scaled by 2^(3-e) (exact) and rounded to an integer r; the code
 * is then (e + 6) * 8 + r, which also carries correctly into the next
 * binade when r reaches 16, and from the subnormals into the normals.
 */
uint8_t tfq_oracle_e4m3_encode(float t)
{
    uint8_t sign = signbit(t) ? 0x80 : 0x00;
    double a;
    int E, e, code;
    if (isnan(t))
        return (uint8_t)(sign | 0x7F);
    a = fabs((double)t);
    if (a > 448.0)
        a = 448.0;
    if (a == 0.0)
        return sign;
    (void)frexp(a, &E); /* a = f * 2^E with f in [0.5, 1) */
    e = E - 1;          /* floor(log2(a)) */
    if (e < -6)
        e = -6;
    code = (e + 6) * 8 + (int)round_half_even_nonneg(ldexp(a, 3 - e));
    if (code > 0x7E)
        code = 0x7E;
    return (uint8_t)(sign | code);
}

/* ------------------------------------------------------------------ */
/* Per-row scale: s = fl32(max(amax, 1e-12) / qmax).                   */
/* ------------------------------------------------------------------ */
static float row_scale(const uint16_t *row, int64_t K, float qmax)
{
    float amax = 0.0f;
    int64_t k;
    for (k = 0; k < K; ++k) {
        float v = fabsf(bf16_bits_to_float(row[k]));
        if (v > amax)
            amax = v;
    }
    if (amax < 1e-12f)
        amax = 1e-12f;
    return amax / qmax;
}

/*
 * Per-row FP8 quantization of a row-major bf16 matrix x[rows, K]:
 *   s[r] = fl32(max(max_k |x[r,k]|, 1e-12) / qmax)
 *   q[r,k] = E4M3FN_RNE(clamp(fl32(x[r,k] / s[r]), -qmax, qmax))
 * Used for per-token activations (rows = tokens) and per-output-channel
 * weights (rows = output channels of an [N, K] weight).
 */
void tfq_oracle_quant_rows_fp8(const uint16_t *x, int64_t rows, int64_t K,
                               float qmax, uint8_t *q, float *s)
{
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; ++r) {
        const uint16_t *row = x + r * K;
        float sc = row_scale(row, K, qmax);
        int64_t k;
        s[r] = sc;
        for (k = 0; k < K; ++k) {
            float t = bf16_bits_to_float(row[k]) / sc;
            if (t > qmax)
                t = qmax;
            if (t < -qmax)
                t = -qmax;
            q[r * K + k] = tfq_oracle_e4m3_encode(t);
        }
    }
}

/*
 * Per-row INT8 quantization (qmax = 127 in the pages' formula):
 *   s[r] = fl32(max(max_k |x[r,k]|, 1e-12) / qmax)
 *   q[r,k] = clamp(round_half_even(fl32(x[r,k] / s[r])), -128, 127)
 */
void tfq_oracle_quant_rows_int8(const uint16_t *x, int64_t rows, int64_t K,
                                float qmax, int8_t *q, float *s)
{
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; ++r) {
        const uint16_t *row = x + r * K;
        float sc = row_scale(row, K, qmax);
        int64_t k;
        s[r] = sc;
        for (k = 0; k < K; ++k) {
            float t = bf16_bits_to_float(row[k]) / sc;
            double mag = round_half_even_nonneg(fabs((double)t));
            double v = (t < 0.0f) ? -mag : mag;
            if (v > 127.0)
                v = 127.0;
            if (v < -128.0)
                v = -128.0;
            q[r * K + k] = (int8_t)v;
        }
    }
}

/*
 * Scaled FP8 GEMM, "TN" layout (both operands K-contiguous):
 *   y[i, n] = (sum_k dec(A[m,k]) * dec(W[n,k])) * s_a[m] * s_w[n] + bias[n]
 * for m = rows[i] (or m = i when rows is NULL), every n in [0, N).
 * bias is a bf16 vector of length N, or NULL for no bias.
 * Output is double, not rounded to bf16.
 */
void tfq_oracle_scaled_fp8_linear(const uint8_t *A, const float *s_a,
                                  const uint8_t *W, const float *s_w,
                                  const uint16_t *bias, int64_t M, int64_t N,
                                  int64_t K, const int64_t *rows,
                                  int64_t nrows, double *y)
{
    double dec[256];
    int64_t i;
    int c;
    (void)M;
    for (c = 0; c < 256; ++c)
        dec[c] = tfq_oracle_e4m3_decode((uint8_t)c);
#pragma omp parallel for schedule(dynamic, 1)
    for (i = 0; i < nrows; ++i) {
        int64_t m = rows ? rows[i] : i;
        const uint8_t *a = A + m * K;
        int64_t n;
        for (n = 0; n < N; ++n) {
            const uint8_t *w = W + n * K;
            double acc = 0.0;
            int64_t k;
            for (k = 0; k < K; ++k)
                acc += dec[a[k]] * dec[w[k]];
            acc = acc * (double)s_a[m] * (double)s_w[n];
            if (bias)
                acc += (double)bf16_bits_to_float(bias[n]);
            y[i * N + n] = acc;
        }
    }
}

/*
 * INT8 x INT8 scaled GEMM with the same epilogue (per-token activation
 * scales, per-output-channel weight scales): the int8-vllm / int8-sgl /
 * int8-torchao modes of the LightX2V "模型量化技术" page, quantization-mode
 * table.  The integer sum is exact in int64.
 */
void tfq_oracle_scaled_int8_linear(const int8_t *A, const float *s_a,
                                   const int8_t *W, const float *s_w,
                                   const uint16_t *bias, int64_t M, int64_t N,
                                   int64_t K, const int64_t *rows,
                                   int64_t nrows, double *y)
{
    int64_t i;
    (void)M;
#pragma omp parallel for schedule(dynamic, 1)
    for (i = 0; i < nrows; ++i) {
        int64_t m = rows ? rows[i] : i;
        const int8_t *a = A + m * K;
        int64_t n;
        for (n = 0; n < N; ++n) {
            const int8_t *w = W + n * K;
            int64_t acc = 0;
            int64_t k;
            double v;
            for (k = 0; k < K; ++k)
                acc += (int64_t)a[k] * (int64_t)w[k];
            v = (double)acc * (double)s_a[m] * (double)s_w[n];
            if (bias)
                v += (double)bf16_bits_to_float(bias[n]);
            y[i * N + n] = v;
        }
    }
}

/*
 * Block prefix sums of the FP8 GEMM's accumulation, for the FP16-accumulator
 * study (LightX2V "模型量化技术" page, section "MiniMax-H3 FP8 FP16 累加":
 * with FP16 accumulation the partial sums of the FFN-out Linear overflow at
 * qmax 14 and 12; qmax 7 keeps them in range).  For m = rows[i] (or i) and
 * every n, with P_j = sum_{k < j * block} dec(A[m,k]) dec(W[n,k]) (exact in
 * double, see above) and P_last the whole sum:
 *   final[i, n]      = P_last,
 *   prefix_max[i, n] = max |P_j| over j = 1 .. ceil(K / block) (the last
 *                      block may be partial), i.e. the largest magnitude the
 *                      running sum reaches at a block boundary.
 * No scales, no bias: these are the accumulator's values.
 */
void tfq_oracle_fp8_block_prefix_sums(const uint8_t *A, const uint8_t *W,
                                      int64_t M, int64_t N, int64_t K,
                                      int64_t block, const int64_t *rows,
                                      int64_t nrows, double *final_sum,
                                      double *prefix_max)
{
    double dec[256];
    int64_t i;
    int c;
    (void)M;
    for (c = 0; c < 256; ++c)
        dec[c] = tfq_oracle_e4m3_decode((uint8_t)c);
#pragma omp parallel for schedule(dynamic, 1)
    for (i = 0; i < nrows; ++i) {
        int64_t m = rows ? rows[i] : i;
        const uint8_t *a = A + m * K;
        int64_t n;
        for (n = 0; n < N; ++n) {
            const uint8_t *w = W + n * K;
            double acc = 0.0, pmax = 0.0;
            int64_t k;
            for (k = 0; k < K; ++k) {
                acc = acc + dec[a[k]] * dec[w[k]];
                if ((k + 1) % block == 0 || k + 1 == K) {
                    if (fabs(acc) > pmax)
                        pmax = fabs(acc);
                }
            }
            final_sum[i * N + n] = acc;
            prefix_max[i * N + n] = pmax;
        }
    }
}

/* ------------------------------------------------------------------ */
/* MXFP8: E4M3 elements with one E8M0 (power-of-two) scale per block of */
/* 32 consecutive values of a row.                                     */
/* ------------------------------------------------------------------ */
/*
 * The TeleFuser "Quantization" page (section "Offline conversion") names the
 * format -- 32-value blocks with E8M0 scales -- but not the conversion.  The
 * reading taken is the conversion of the OCP Microscaling Formats (MX) v1.0
 * specification (section "Conversion from vectors of scalars to MX"):
 *   shared exponent  E = floor(log2(max_k |x_k|)) - emax,  emax = 8 for E4M3
 *                    (its largest normal is 1.75 * 2^8 = 448);
 *   E is clamped to the E8M0 range [-127, 127] and stored as code E + 127;
 *   element          q_k = E4M3_RNE(clamp(x_k / 2^E, -448, 448)).
 * A block whose values are all zero has no exponent; it takes the smallest
 * scale, code 0 (its elements are zeros whatever the scale).
 * Dividing by 2^E is exact in double, so no fp32 rounding step is involved.
 */
static uint8_t e8m0_block_code(float amax)
{
    int E, e;
    if (amax == 0.0f)
        return 0;
    (void)frexp((double)amax, &E); /* amax = f * 2^E, f in [0.5, 1) */
    e = (E - 1) - 8;               /* floor(log2(amax)) - emax(E4M3) */
    if (e < -127)
        e = -127;
    if (e > 127)
        e = 127;
    return (uint8_t)(e + 127);
}

/*
 * MXFP8 quantization of a row-major bf16 matrix x[rows, K] (K % 32 == 0):
 * codes q[rows, K] and scale codes sf[rows, K / 32], both row-major.  Used
 * for activations (rows = tokens) and weights (rows = output channels).
 */
void tfq_oracle_quant_mxfp8(const uint16_t *x, int64_t rows, int64_t K,
                            uint8_t *q, uint8_t *sf)
{
    const int64_t nb = K / 32;
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; ++r) {
        int64_t b;
        for (b = 0; b < nb; ++b) {
            const uint16_t *blk = x + r * K + b * 32;
            float amax = 0.0f;
            uint8_t code;
            double scale;
            int k;
            for (k = 0; k < 32; ++k) {
                float v = fabsf(bf16_bits_to_float(blk[k]));
                if (v > amax)
                    amax = v;
            }
            code = e8m0_block_code(amax);
            sf[r * nb + b] = code;
            scale = ldexp(1.0, (int)code - 127);
            for (k = 0; k < 32; ++k) {
                double t = (double)bf16_bits_to_float(blk[k]) / scale;
                if (t > 448.0)
                    t = 448.0;
                if (t < -448.0)
                    t = -448.0;
                q[r * K + b * 32 + k] = tfq_oracle_e4m3_encode((float)t);
            }
        }
    }
}

/*
 * MXFP8 GEMM, "TN" layout, both operands block-scaled along K:
 *   y[i, n] = sum_b 2^(sfa[m,b] - 127) * 2^(sfw[n,b] - 127)
 *                   * sum_{k in block b} dec(A[m,k]) * dec(W[n,k])   (+ bias[n])
 * for m = rows[i] (or m = i when rows is NULL).  Each block sum is exact in
 * double (32 products, each a multiple of 2^-18 below 2^18); the power-of-two
 * scaling is exact; only the sum over blocks rounds (to 53 bits).
 */
void tfq_oracle_mxfp8_linear(const uint8_t *A, const uint8_t *sfa,
                             const uint8_t *W, const uint8_t *sfw,
                             const uint16_t *bias, int64_t M, int64_t N,
                             int64_t K, const int64_t *rows, int64_t nrows,
                             double *y)
{
    const int64_t nb = K / 32;
    double dec[256];
    int64_t i;
    int c;
    (void)M;
    for (c = 0; c < 256; ++c)
        dec[c] = tfq_oracle_e4m3_decode((uint8_t)c);
#pragma omp parallel for schedule(dynamic, 1)
    for (i = 0; i < nrows; ++i) {
        int64_t m = rows ? rows[i] : i;
        int64_t n;
        for (n = 0; n < N; ++n) {
            double acc = 0.0;
            int64_t b;
            for (b = 0; b < nb; ++b) {
                const uint8_t *a = A + m * K + b * 32;
                const uint8_t *w = W + n * K + b * 32;
                double part = 0.0;
                int k;
                for (k = 0; k < 32; ++k)
                    part += dec[a[k]] * dec[w[k]];
                acc += ldexp(part, (int)sfa[m * nb + b] + (int)sfw[n * nb + b] - 254);
            }
            if (bias)
                acc += (double)bf16_bits_to_float(bias[n]);
            y[i * N + n] = acc;
        }
    }
}

/* Threads the OpenMP loops above use (1 when built without OpenMP). */
int tfq_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void tfq_oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}
