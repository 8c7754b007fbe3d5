// tfq_quant.cu -- per-row absmax quantizer (BF16 -> E4M3FN or INT8 + fp32
// scale per row), HBM-bandwidth bound.
//
// Computes, for every row r of a row-major bf16 matrix x[rows, K]:
//   s[r]   = fl32(max(max_k |x[r,k]|, 1e-12) / qmax)
//   q[r,k] = E4M3FN_rn_satfinite(clamp(fl32(x[r,k] / s[r]), -qmax, qmax))     (FP8)
//   q[r,k] = clamp(rint_half_even(fl32(x[r,k] / s[r])), -128, 127)             (INT8)
// which is the per-row scaled-FP8 formula of the TeleFuser "Quantization"
// page (section "Scaled FP8 checkpoints: W8A8"), with the reduced qmax of
// the LightX2V "模型量化技术" page (section "MiniMax-H3 FP8 FP16 累加"), and
// the symmetric INT8 formula of the TeleFuser page (section "Core ideas").
// Rows are tokens (activations) or output channels (weights).
//
// Design (B200): each CTA is persistent over groups of consecutive rows.
// One producer thread streams row groups HBM -> shared memory with 1-D bulk
// copies (cp.async.bulk, completion on an mbarrier) into a ring of stages,
// so tens of KB per SM are in flight with a single issuing thread.  Eight
// consumer warps split each stage: a "team" of 1, 2, 4 or 8 warps owns one
// row, reduces |x| with packed bf16x2 max + warp shuffles (and, for teams
// larger than one warp, an mbarrier-synchronised exchange through shared
// memory), then re-reads the row from shared memory, divides, converts two
// values per cvt instruction and stores 8 output bytes per thread per step
// (a warp writes 256 contiguous bytes).  Every wait is bounded.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>

#include "tfq_internal.h"
#include "tfq_ptx.cuh"

namespace tfq {
namespace {

constexpr int kComputeWarps = 8;
constexpr int kThreads = (kComputeWarps + 1) * 32;  // + one producer warp
#ifndef TFQ_QUANT_STAGE_KB
#define TFQ_QUANT_STAGE_KB 32   // bytes of x per stage (target), KiB
#endif
#ifndef TFQ_QUANT_RING_KB
#define TFQ_QUANT_RING_KB 72    // ring size target per CTA, KiB (three CTAs per SM)
#endif
#ifndef TFQ_QUANT_CTAS_PER_SM
#define TFQ_QUANT_CTAS_PER_SM 3
#endif
constexpr uint32_t kStageTarget = TFQ_QUANT_STAGE_KB * 1024;
constexpr uint32_t kSmemTarget = TFQ_QUANT_RING_KB * 1024;
constexpr uint32_t kBulkPiece = 32 * 1024;          // one cp.async.bulk moves at most this

struct QuantConfig {
    int rows_per_stage;
    int warps_per_row;  // team size: 1, 2, 4 or 8
    int stages;
    uint32_t stage_bytes;
    uint32_t smem_bytes;
};

__host__ QuantConfig choose_config(int64_t K) {
    QuantConfig c{};
    const uint32_t row_bytes = static_cast<uint32_t>(2 * K);
    int r = static_cast<int>(std::max<uint32_t>(1u, kStageTarget / row_bytes));
    if (r >= 8) {
        c.warps_per_row = 1;
        c.rows_per_stage = std::min(r, 64);
    } else if (r >= 4) {
        c.warps_per_row = 2;
        c.rows_per_stage = 4;
    } else if (r >= 2) {
        c.warps_per_row = 4;
        c.rows_per_stage = 2;
    } else {
        c.warps_per_row = 8;
        c.rows_per_stage = 1;
    }
    c.stage_bytes = (static_cast<uint32_t>(c.rows_per_stage) * row_bytes + 127u) & ~127u;
    c.stages = static_cast<int>(std::min<uint32_t>(8u, std::max<uint32_t>(2u, kSmemTarget / c.stage_bytes)));
    // ring + full/empty barriers + team barriers + amax exchange + abort flag
    c.smem_bytes = c.stages * c.stage_bytes + 2 * c.stages * 8 + kComputeWarps * 8 + 2 * kComputeWarps * 4 + 16;
    return c;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Packed max of magnitudes: each bf16 half of the result has magnitude
// max(|a|, |b|) (its sign bit is the XOR of the inputs' signs and is ignored).
__device__ __forceinline__ uint32_t max_abs_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Two fp32 values -> two E4M3FN codes (round to nearest even, saturate to
// +-448): `lo` goes to the low byte, `hi` to the high byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tmov.b16 %0, t;\n\t}"
        : "=h"(r)
        : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t to_int8_byte(float t) {
    int i = __float2int_rn(t);  // round half to even
    i = min(max(i, -128), 127);
    return static_cast<uint32_t>(i) & 0xFFu;
}

}  // namespace

// Correctly rounded fp32 quotient a / b, given y = RN(1/b), by Markstein's
// method (P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): if y is the
// correctly rounded reciprocal of b and q is a faithful approximation of
// a/b, then r = a - b*q is exact in one FMA and RN(q + r*y) = RN(a/b).
// q0 = RN(a*y) is within 1.5 ulp of a/b; one correction step makes it
// faithful (q1 is within 1/2 ulp plus a term of order 2^-23 ulp), the
// second step rounds it correctly.  The argument needs y and the residuals
// to be normal numbers, which holds for |a| >= 2^-102 and
// 2^-49 <= b <= 2^125 (every row scale is >= 1e-12 / 448 > 2^-49; rows with
// a larger scale take the IEEE division instead).  For |a| < 2^-102 the
// quotient is below 2^-53 in magnitude, so only its sign reaches the codes;
// the final copysign keeps it, also for a = +-0.  Five FMA-pipe
// instructions, no branch.  Checked against the IEEE division __fdiv_rn by
// tfq_selftest_div_rn.
__device__ __forceinline__ float div_rn_from_rcp(float a, float b, float y) {
    const float q0 = __fmul_rn(a, y);
    const float r0 = __fmaf_rn(-q0, b, a);
    const float q1 = __fmaf_rn(r0, y, q0);
    const float r1 = __fmaf_rn(-q1, b, a);
    const float q2 = __fmaf_rn(r1, y, q1);
    return copysignf(q2, a);
}

namespace {

// Quantizes the 8 bf16 values of `v` with scale `sc` (rcp = RN(1/sc)): 8
// output bytes.  kClamp: clamp x/s to +-qmax before the cast.  The clamp is
// skipped when qmax is an E4M3 value: then |x/s| <= qmax + 1 ulp(qmax)
// (s = RN(amax/qmax) and |x| <= amax), and qmax + 1 ulp encodes like qmax
// because the nearest E4M3 midpoint is 2^-4 of a binade away (448 + ulp
// saturates to 448).
template <bool kInt8, bool kClamp, bool kIeeeDiv>
__device__ __forceinline__ uint2 quantize8(uint4 v, float sc, float rcp, float qmax) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t packed[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float a, b;
        if constexpr (kIeeeDiv) {
            a = __fdiv_rn(bf16_lo(w[j]), sc);
            b = __fdiv_rn(bf16_hi(w[j]), sc);
        } else {
            a = div_rn_from_rcp(bf16_lo(w[j]), sc, rcp);
            b = div_rn_from_rcp(bf16_hi(w[j]), sc, rcp);
        }
        if constexpr (kInt8) {
            packed[j] = to_int8_byte(a) | (to_int8_byte(b) << 8);
        } else {
            if constexpr (kClamp) {
                a = fminf(fmaxf(a, -qmax), qmax);
                b = fminf(fmaxf(b, -qmax), qmax);
            }
            packed[j] = cvt_e4m3x2(a, b);
        }
    }
    return make_uint2(packed[0] | (packed[1] << 16), packed[2] | (packed[3] << 16));
}

__device__ __forceinline__ void record_failure(volatile int* abort_flag, uint32_t* err, uint32_t bit) {
    *abort_flag = 1;
    atomicOr(err, bit);
}

template <bool kInt8, bool kClamp>
__global__ void __launch_bounds__(kThreads) quant_rows_kernel(const uint16_t* __restrict__ x, int64_t M, int K,
                                                              float qmax, uint8_t* __restrict__ q,
                                                              float* __restrict__ s, QuantConfig cfg,
                                                              uint32_t* err) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int S = cfg.stages;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(S) * cfg.stage_bytes);
    uint64_t* empty = full + S;
    uint64_t* team_bar = empty + S;                               // one per row slot
    float* red = reinterpret_cast<float*>(team_bar + kComputeWarps);  // [2][8]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(red + 2 * kComputeWarps);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int R = cfg.rows_per_stage;
    const int G = cfg.warps_per_row;
    const int64_t n_groups = (M + R - 1) / R;
    const uint32_t row_bytes = 2u * static_cast<uint32_t>(K);

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kComputeWarps);
        }
        for (int i = 0; i < kComputeWarps; ++i) mbar_init(&team_bar[i], G);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kComputeWarps) {
        // ------------------------------------------------------- producer
        if (lane != 0) return;
        int issued_phase[8];
        for (int i = 0; i < 8; ++i) issued_phase[i] = -1;
        int it = 0;
        for (int64_t g = blockIdx.x; g < n_groups; g += gridDim.x, ++it) {
            const int st = it % S;
            const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
            if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag)) {
                record_failure(abort_flag, err, kErrQuantProducer);
                break;
            }
            const int64_t r0 = g * R;
            const uint32_t rows = static_cast<uint32_t>(min(static_cast<int64_t>(R), M - r0));
            const uint32_t bytes = rows * row_bytes;
            mbar_arrive_expect_tx(&full[st], bytes);
            const uint8_t* src = reinterpret_cast<const uint8_t*>(x + r0 * K);
            uint8_t* dst = smem + static_cast<size_t>(st) * cfg.stage_bytes;
            for (uint32_t off = 0; off < bytes; off += kBulkPiece)
                bulk_g2s(dst + off, src + off, min(kBulkPiece, bytes - off), &full[st]);
            issued_phase[st] = static_cast<int>(ph);
        }
        // Every copy this thread issued must land before the CTA may exit
        // (on the normal path they already have, or soon will).
        for (int i = 0; i < S; ++i) {
            if (issued_phase[i] >= 0 && !mbar_wait(&full[i], static_cast<uint32_t>(issued_phase[i]), nullptr))
                atomicOr(err, kErrQuantProducer);
        }
        return;
    }

    // ------------------------------------------------------------ consumers
    const int slot = warp / G;
    const int nslots = kComputeWarps / G;
    const int tr = (warp % G) * 32 + lane;  // index within the row team
    const int team = G * 32;
    const int units = K / 8;                // 16-byte units of 8 bf16
    uint32_t team_uses = 0;
    int it = 0;
    for (int64_t g = blockIdx.x; g < n_groups; g += gridDim.x, ++it) {
        const int st = it % S;
        const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
        if (!mbar_wait_warp(&full[st], ph, abort_flag)) {
            if (lane == 0) record_failure(abort_flag, err, kErrQuantConsumer);
            break;
        }
        const int64_t r0 = g * R;
        const int rows = static_cast<int>(min(static_cast<int64_t>(R), M - r0));
        const uint8_t* stage = smem + static_cast<size_t>(st) * cfg.stage_bytes;
        bool ok = true;
        for (int r = slot; r < rows; r += nslots) {
            const uint4* row = reinterpret_cast<const uint4*>(stage + static_cast<size_t>(r) * row_bytes);
            // pass 1: max |x| (bf16 magnitudes, packed)
            uint32_t m2 = 0, m3 = 0;
#pragma unroll 4
            for (int u = tr; u < units; u += team) {
                const uint4 v = row[u];
                m2 = max_abs_bf16x2(m2, v.x);
                m3 = max_abs_bf16x2(m3, v.y);
                m2 = max_abs_bf16x2(m2, v.z);
                m3 = max_abs_bf16x2(m3, v.w);
            }
            m2 = max_abs_bf16x2(m2, m3) & 0x7FFF7FFFu;
            float amax = fmaxf(bf16_lo(m2), bf16_hi(m2));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
            if (G > 1) {
                float* red_buf = red + (team_uses & 1u) * kComputeWarps;
                if (lane == 0) {
                    red_buf[warp] = amax;
                    mbar_arrive(&team_bar[slot]);
                }
                __syncwarp();
                if (!mbar_wait_warp(&team_bar[slot], team_uses & 1u, abort_flag)) {
                    if (lane == 0) record_failure(abort_flag, err, kErrQuantConsumer);
                    ok = false;
                    break;
                }
                amax = red_buf[slot * G];
                for (int j = 1; j < G; ++j) amax = fmaxf(amax, red_buf[slot * G + j]);
                ++team_uses;
            }
            const float sc = __fdiv_rn(fmaxf(amax, 1e-12f), qmax);
            const float rcp = __frcp_rn(sc);
            const int64_t grow = r0 + r;
            if (tr == 0) s[grow] = sc;
            // pass 2: quantize and store (8 bytes per thread, 256 B per warp)
            uint2* qrow = reinterpret_cast<uint2*>(q + grow * K);
            if (sc <= 0x1p125f) {
#pragma unroll 2
                for (int u = tr; u < units; u += team)
                    qrow[u] = quantize8<kInt8, kClamp, false>(row[u], sc, rcp, qmax);
            } else {  // reciprocal would be subnormal: IEEE division (row-uniform branch)
                for (int u = tr; u < units; u += team)
                    qrow[u] = quantize8<kInt8, kClamp, true>(row[u], sc, rcp, qmax);
            }
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
    }
}

// Element-wise self-check of div_rn_from_rcp against the IEEE division.
__global__ void div_selftest_kernel(const float* __restrict__ a, const float* __restrict__ b, int64_t n,
                                    float* __restrict__ ours, float* __restrict__ ieee) {
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float x = a[i], y = b[i];
        ours[i] = div_rn_from_rcp(x, y, __frcp_rn(y));
        ieee[i] = __fdiv_rn(x, y);
    }
}

// K == 0: an empty row has amax 0, so only the floored scale is written.
__global__ void empty_rows_scale_kernel(int64_t M, float qmax, float* s) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < M) s[i] = __fdiv_rn(1e-12f, qmax);
}

// True when v is exactly representable in E4M3FN (at most 4 significant bits,
// within the normal range used for qmax).
bool is_e4m3_value(float v) {
    int e = 0;
    const float m = std::frexp(v, &e) * 16.0f;  // 4 significant bits -> integer
    return v >= 0x1p-6f && v <= 448.0f && m == std::floor(m);
}

}  // namespace

tfq_status launch_div_selftest(const float* a, const float* b, int64_t n, float* ours, float* ieee,
                               cudaStream_t stream) {
    if (n == 0) return TFQ_OK;
    const int threads = 256;
    const int64_t blocks = std::min<int64_t>((n + threads - 1) / threads, 65535);
    div_selftest_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(a, b, n, ours, ieee);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TFQ_OK : fail(TFQ_ECUDA, "self-test launch: %s", cudaGetErrorString(e));
}

tfq_status launch_quant_rows(const void* x, int64_t rows, int64_t K, float qmax, bool out_int8, void* q, float* s,
                             cudaStream_t stream, DeviceState* ds) {
    if (rows == 0) return TFQ_OK;
    if (K == 0) {
        const int threads = 256;
        const int64_t blocks = (rows + threads - 1) / threads;
        empty_rows_scale_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(rows, qmax, s);
        const cudaError_t e = cudaGetLastError();
        return e == cudaSuccess ? TFQ_OK : fail(TFQ_ECUDA, "quantizer launch: %s", cudaGetErrorString(e));
    }
    const QuantConfig cfg = choose_config(K);
    const bool clamp = !out_int8 && !is_e4m3_value(qmax);
    auto kernel = out_int8 ? quant_rows_kernel<true, false>
                           : (clamp ? quant_rows_kernel<false, true> : quant_rows_kernel<false, false>);
    const int kidx = out_int8 ? 2 : (clamp ? 1 : 0);
    if (!ds->quant_attr_set[kidx]) {
        const cudaError_t e =
            cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (e != cudaSuccess) return fail(TFQ_ECUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        ds->quant_attr_set[kidx] = true;
    }
    const int64_t n_groups = (rows + cfg.rows_per_stage - 1) / cfg.rows_per_stage;
    const int per_sm = std::max(1, static_cast<int>((228u * 1024u) / (cfg.smem_bytes + 1024u)));
    const int64_t grid = std::min<int64_t>(n_groups, static_cast<int64_t>(ds->sm_count) * std::min(per_sm, TFQ_QUANT_CTAS_PER_SM));
    kernel<<<static_cast<unsigned>(grid), kThreads, cfg.smem_bytes, stream>>>(
        static_cast<const uint16_t*>(x), rows, static_cast<int>(K), qmax, static_cast<uint8_t*>(q), s, cfg,
        ds->err_word);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TFQ_OK : fail(TFQ_ECUDA, "quantizer launch: %s", cudaGetErrorString(e));
}

}  // namespace tfq
