/*
 * A W8A8 Linear driven from plain C through include/tfq.h, with device
 * memory from the CUDA runtime and no Python anywhere: per-token FP8
 * quantization of bf16 activations, per-channel FP8 quantization of two
 * weights, and both Linears as one multi-Linear GEMM (as Q and K of a DiT
 * block read one input).  The results are checked against the CPU oracle
 * (oracle/tfq_oracle.c, linked as liboracle.so): codes and scales bit for
 * bit, each output within |y - y_ref| <= 2^-7 |y_ref| + 1e-3 rms(y_ref).
 *
 * Exit status 0 and "ok" on success, 1 with a message otherwise.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "tfq.h"

/* The oracle's entry points (test infrastructure; see oracle/tfq_oracle.c). */
void tfq_oracle_quant_rows_fp8(const uint16_t *x, int64_t rows, int64_t K, float qmax, uint8_t *q, float *s);
void tfq_oracle_scaled_fp8_linear(const uint8_t *A, const float *s_a, const uint8_t *W, const float *s_w,
                                  const uint16_t *bias, int64_t M, int64_t N, int64_t K, const int64_t *rows,
                                  int64_t nrows, double *y);

enum { M = 700, K = 512, N0 = 264, N1 = 1032 };

static uint64_t rng_state = 0x9E3779B97F4A7C15ull;

/* xorshift64*: a uniform double in [0, 1) */
static double uniform(void) {
    rng_state ^= rng_state >> 12;
    rng_state ^= rng_state << 25;
    rng_state ^= rng_state >> 27;
    return (double)((rng_state * 0x2545F4914F6CDD1Dull) >> 11) * 0x1.0p-53;
}

/* bf16 bits of a float (round to nearest even; inputs here are finite) */
static uint16_t to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

static float from_bf16(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static void fill(uint16_t *x, size_t n, double scale) {
    for (size_t i = 0; i < n; ++i) x[i] = to_bf16((float)((uniform() * 2.0 - 1.0) * scale));
}

static int fail(const char *what) {
    fprintf(stderr, "FAIL: %s\n", what);
    return 1;
}

#define CUDA(call)                                                                     \
    do {                                                                               \
        cudaError_t e_ = (call);                                                       \
        if (e_ != cudaSuccess) {                                                       \
            fprintf(stderr, "FAIL: %s: %s\n", #call, cudaGetErrorString(e_));          \
            return 1;                                                                  \
        }                                                                              \
    } while (0)

#define TFQ(call)                                                                                        \
    do {                                                                                                 \
        tfq_status s_ = (call);                                                                          \
        if (s_ != TFQ_OK) {                                                                              \
            fprintf(stderr, "FAIL: %s: %s: %s\n", #call, tfq_status_string(s_), tfq_last_error_message()); \
            return 1;                                                                                    \
        }                                                                                                \
    } while (0)

static int check_linear(const char *name, const uint16_t *y, const double *ref, int64_t n) {
    double ss = 0.0, worst = 0.0;
    for (int64_t i = 0; i < n; ++i) ss += ref[i] * ref[i];
    const double rms = sqrt(ss / (double)n);
    for (int64_t i = 0; i < n; ++i) {
        const double err = fabs((double)from_bf16(y[i]) - ref[i]);
        const double bound = 0x1.0p-7 * fabs(ref[i]) + 1e-3 * rms;
        if (!(err <= bound)) {
            fprintf(stderr, "FAIL: %s element %lld: %g vs %g\n", name, (long long)i, (double)from_bf16(y[i]), ref[i]);
            return 1;
        }
        if (err / bound > worst) worst = err / bound;
    }
    printf("%s: worst error / bound %.3f\n", name, worst);
    return 0;
}

int main(void) {
    const int64_t Ns[2] = {N0, N1};
    uint16_t *hx = malloc(sizeof(uint16_t) * M * K);
    uint16_t *hw[2], *hb[2];
    for (int i = 0; i < 2; ++i) {
        hw[i] = malloc(sizeof(uint16_t) * Ns[i] * K);
        hb[i] = malloc(sizeof(uint16_t) * Ns[i]);
    }
    if (hx == NULL || hw[0] == NULL || hw[1] == NULL || hb[0] == NULL || hb[1] == NULL) return fail("host malloc");
    fill(hx, (size_t)M * K, 3.0);
    for (int i = 0; i < 2; ++i) {
        fill(hw[i], (size_t)Ns[i] * K, 0.05);
        fill(hb[i], (size_t)Ns[i], 0.5);
    }

    void *dx, *dA, *dW[2], *dWq[2], *db[2], *dy[2];
    float *dsa, *dsw[2];
    CUDA(cudaMalloc(&dx, sizeof(uint16_t) * M * K));
    CUDA(cudaMalloc(&dA, (size_t)M * K));
    CUDA(cudaMalloc((void **)&dsa, sizeof(float) * M));
    CUDA(cudaMemcpy(dx, hx, sizeof(uint16_t) * M * K, cudaMemcpyHostToDevice));
    for (int i = 0; i < 2; ++i) {
        CUDA(cudaMalloc(&dW[i], sizeof(uint16_t) * Ns[i] * K));
        CUDA(cudaMalloc(&dWq[i], (size_t)Ns[i] * K));
        CUDA(cudaMalloc((void **)&dsw[i], sizeof(float) * Ns[i]));
        CUDA(cudaMalloc(&db[i], sizeof(uint16_t) * Ns[i]));
        CUDA(cudaMalloc(&dy[i], sizeof(uint16_t) * M * Ns[i]));
        CUDA(cudaMemcpy(dW[i], hw[i], sizeof(uint16_t) * Ns[i] * K, cudaMemcpyHostToDevice));
        CUDA(cudaMemcpy(db[i], hb[i], sizeof(uint16_t) * Ns[i], cudaMemcpyHostToDevice));
        TFQ(tfq_quant_weight_per_channel(dW[i], Ns[i], K, TFQ_DTYPE_FP8_E4M3, 448.0f, dWq[i], dsw[i], NULL));
    }
    TFQ(tfq_quant_act_fp8_per_token(dx, M, K, 448.0f, dA, dsa, NULL));
    const void *W_q[2] = {dWq[0], dWq[1]};
    const float *s_w[2] = {dsw[0], dsw[1]};
    const void *bias[2] = {db[0], db[1]};
    void *out[2] = {dy[0], dy[1]};
    TFQ(tfq_scaled_fp8_linear_multi(dA, dsa, M, K, 2, W_q, s_w, bias, Ns, out, NULL));
    CUDA(cudaDeviceSynchronize());
    TFQ(tfq_device_error(NULL));

    /* codes and scales against the oracle */
    uint8_t *A = malloc((size_t)M * K), *A_ref = malloc((size_t)M * K);
    float *sa = malloc(sizeof(float) * M), *sa_ref = malloc(sizeof(float) * M);
    if (A == NULL || A_ref == NULL || sa == NULL || sa_ref == NULL) return fail("host malloc");
    CUDA(cudaMemcpy(A, dA, (size_t)M * K, cudaMemcpyDeviceToHost));
    CUDA(cudaMemcpy(sa, dsa, sizeof(float) * M, cudaMemcpyDeviceToHost));
    tfq_oracle_quant_rows_fp8(hx, M, K, 448.0f, A_ref, sa_ref);
    if (memcmp(A, A_ref, (size_t)M * K) != 0) return fail("activation codes differ from the oracle");
    if (memcmp(sa, sa_ref, sizeof(float) * M) != 0) return fail("activation scales differ from the oracle");
    for (int i = 0; i < 2; ++i) {
        const int64_t n = Ns[i];
        uint8_t *Wq = malloc((size_t)n * K), *Wq_ref = malloc((size_t)n * K);
        float *sw = malloc(sizeof(float) * n), *sw_ref = malloc(sizeof(float) * n);
        uint16_t *y = malloc(sizeof(uint16_t) * M * n);
        double *y_ref = malloc(sizeof(double) * M * n);
        if (Wq == NULL || Wq_ref == NULL || sw == NULL || sw_ref == NULL || y == NULL || y_ref == NULL)
            return fail("host malloc");
        CUDA(cudaMemcpy(Wq, dWq[i], (size_t)n * K, cudaMemcpyDeviceToHost));
        CUDA(cudaMemcpy(sw, dsw[i], sizeof(float) * n, cudaMemcpyDeviceToHost));
        CUDA(cudaMemcpy(y, dy[i], sizeof(uint16_t) * M * n, cudaMemcpyDeviceToHost));
        tfq_oracle_quant_rows_fp8(hw[i], n, K, 448.0f, Wq_ref, sw_ref);
        if (memcmp(Wq, Wq_ref, (size_t)n * K) != 0 || memcmp(sw, sw_ref, sizeof(float) * n) != 0)
            return fail("weight codes or scales differ from the oracle");
        tfq_oracle_scaled_fp8_linear(A_ref, sa_ref, Wq_ref, sw_ref, hb[i], M, n, K, NULL, M, y_ref);
        if (check_linear(i == 0 ? "Linear 0" : "Linear 1", y, y_ref, (int64_t)M * n)) return 1;
        free(Wq), free(Wq_ref), free(sw), free(sw_ref), free(y), free(y_ref);
        CUDA(cudaFree(dW[i]));
        CUDA(cudaFree(dWq[i]));
        CUDA(cudaFree(dsw[i]));
        CUDA(cudaFree(db[i]));
        CUDA(cudaFree(dy[i]));
        free(hw[i]), free(hb[i]);
    }
    CUDA(cudaFree(dx));
    CUDA(cudaFree(dA));
    CUDA(cudaFree(dsa));
    free(hx), free(A), free(A_ref), free(sa), free(sa_ref);
    printf("ok\n");
    return 0;
}
