// tfq_quant_mx.cu -- MXFP8 block quantizer: BF16 -> E4M3FN codes with one
// E8M0 scale per 32 consecutive elements of a row, written in the
// scale-factor layout the block-scaled tensor-core MMA reads (include/tfq.h).
// The TeleFuser "Quantization" page (section "Offline conversion") names the
// format; the conversion is the one of the OCP Microscaling (MX) v1.0
// specification.  HBM-bandwidth bound.
#include <algorithm>

#include "tfq_internal.h"
#include "tfq_quant_common.cuh"

namespace tfq {
namespace {

// ------------------------------------------------------------------ MXFP8
// One E8M0 scale per 32 consecutive elements of a row (the OCP MX v1.0
// conversion): E = floor(log2(block max)) - 8, clamped to [-127, 127], code
// E + 127 (0 for a block of zeros); q = E4M3_rn_satfinite(x * 2^-E).  The
// product with the power of two is exact (it only rounds when the result is
// far below the smallest E4M3 subnormal, where the code is a signed zero
// anyway), so no division is needed.
//
// The work unit is one 512-byte atom of the scale-factor layout: 128 rows x
// 128 columns of x (4 blocks per row).  Inside an atom, row r owns the word
// 4 ((r % 128) / 32) of the 16-byte line r % 32, so the 16 rows
// {4w .. 4w+3} + {0, 32, 64, 96} own lines 4w .. 4w+3: 64 contiguous bytes.
// Warp w of a CTA takes exactly those rows, two per load instruction (16
// lanes x 16 bytes = one row's 128 columns), all 16 in flight at once; a
// block is 4 adjacent lanes (maximum in two shuffles), and each row's four
// codes leave as one 32-bit word.  Every line of codes and of scales is thus
// written whole by one warp -- no partially written sectors for the memory
// system to merge -- and the padding entries (rows past `rows`, blocks past
// K / 32) come out of the same loop with code 127.

__device__ __forceinline__ uint32_t e8m0_code(float amax) {
    const uint32_t bits = __float_as_uint(amax);
    if (bits == 0u) return 0u;
    const int biased = static_cast<int>(bits >> 23);
    // floor(log2(amax)): from the exponent field, or for a subnormal from the
    // position of the leading mantissa bit (value m * 2^-149)
    const int fl = biased != 0 ? biased - 127 : -118 - __clz(bits);
    return static_cast<uint32_t>(min(max(fl + 119, 0), 254));
}

// 2^(127 - code) as fp32; code 254 gives 2^-127, a subnormal.
__device__ __forceinline__ float e8m0_inverse(uint32_t code) {
    const int k = 127 - static_cast<int>(code);
    return k >= -126 ? __uint_as_float(static_cast<uint32_t>(k + 127) << 23) : __uint_as_float(0x00400000u);
}

__device__ __forceinline__ uint32_t mx_pair(uint32_t w, float2 inv2) {
    const float2 t = __fmul2_rn(make_float2(bf16_lo(w), bf16_hi(w)), inv2);
    return cvt_e4m3x2(t.x, t.y);
}

__device__ __forceinline__ uint2 quantize8_mx(const uint4& v, float inv) {
    const float2 inv2 = make_float2(inv, inv);
    const uint32_t lo = mx_pair(v.x, inv2) | (mx_pair(v.y, inv2) << 16);
    const uint32_t hi = mx_pair(v.z, inv2) | (mx_pair(v.w, inv2) << 16);
    return make_uint2(lo | sign_bytes(v.x, v.y), hi | sign_bytes(v.z, v.w));
}

#ifndef TFQ_MX_CTAS
#define TFQ_MX_CTAS 3  // resident CTAs of 8 warps per SM (~75 registers)
#endif

__global__ void __launch_bounds__(256, TFQ_MX_CTAS) quant_mxfp8_kernel(const uint4* __restrict__ x, int64_t rows,
                                                                       int K, uint8_t* __restrict__ q,
                                                                       uint8_t* __restrict__ sf) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;  // 0..7
    const int half = lane >> 4;         // which of the two rows of a load
    const int lu = lane & 15;           // 16-byte unit within the atom's 128 columns
    const int units = K >> 3;
    const int nb = K >> 5;
    const int64_t ra = (rows + 127) >> 7;
    const int ka_n = (K + 127) >> 7;
    const int64_t tiles = ra * ka_n;
    uint2* q2 = reinterpret_cast<uint2*>(q);
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int64_t rp = t / ka_n;  // 128-row panel
        const int ka = static_cast<int>(t - rp * ka_n);
        const int u = ka * 16 + lu;
        const bool col_ok = u < units;
        uint4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int ri = 2 * j + half;
            const int rl = 4 * warp + (ri & 3) + 32 * (ri >> 2);
            const int64_t r = rp * 128 + rl;
            v[j] = (r < rows && col_ok) ? ldg_nc_v4(x + r * units + u) : make_uint4(0u, 0u, 0u, 0u);
        }
        const bool block_ok = ka * 4 + (lu >> 2) < nb;
        uint8_t* atom = sf + (static_cast<int64_t>(ka) * ra + rp) * 512;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int ri = 2 * j + half;
            const int rl = 4 * warp + (ri & 3) + 32 * (ri >> 2);
            const int64_t r = rp * 128 + rl;
            const uint32_t m = max_abs4(0u, v[j]) & 0x7FFF7FFFu;
            float amax = fmaxf(bf16_lo(m), bf16_hi(m));
            amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
            const bool row_ok = r < rows;
            const uint32_t code = (row_ok && block_ok) ? e8m0_code(amax) : 127u;
            if (row_ok && col_ok) q2[r * units + u] = quantize8_mx(v[j], e8m0_inverse(code));
            // codes of the row's four blocks (lanes 16 half + 0, 4, 8, 12) -> one word
            const uint32_t c1 = __shfl_down_sync(0xFFFFFFFFu, code, 4);
            const uint32_t c2 = __shfl_down_sync(0xFFFFFFFFu, code, 8);
            const uint32_t c3 = __shfl_down_sync(0xFFFFFFFFu, code, 12);
            if (lu == 0)
                *reinterpret_cast<uint32_t*>(atom + 16 * (rl & 31) + 4 * (rl >> 5)) =
                    code | (c1 << 8) | (c2 << 16) | (c3 << 24);
        }
    }
}

}  // namespace

tfq_status launch_quant_mxfp8(const void* x, int64_t rows, int64_t K, void* q, void* sf, cudaStream_t stream,
                              DeviceState* ds) {
    if (rows == 0 || K == 0) return TFQ_OK;
    const int64_t tiles = ((rows + 127) / 128) * ((K + 127) / 128);
    const int64_t blocks = std::min<int64_t>(tiles, static_cast<int64_t>(ds->sm_count) * TFQ_MX_CTAS);
    quant_mxfp8_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const uint4*>(x), rows, static_cast<int>(K), static_cast<uint8_t*>(q), static_cast<uint8_t*>(sf));
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TFQ_OK : fail(TFQ_ECUDA, "quantizer launch: %s", cudaGetErrorString(e));
}

}  // namespace tfq
