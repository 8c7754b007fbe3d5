// tfq_quant_row.cuh -- per-row quantization arithmetic shared by the row
// quantizer kernels (tfq_quant.cu) and the GEMM that quantizes its own
// activations (tfq_gemm.cu): the correctly rounded division x / s, the E4M3
// and INT8 encodings of a 16-byte unit of bf16 values, and one warp's pass
// over a whole row.
//
// What it computes, for a row x[0..K) of bf16 values:
//   s    = fl32(max(max_k |x[k]|, 1e-12) / qmax)
//   q[k] = E4M3FN_rn_satfinite(clamp(fl32(x[k] / s), -qmax, qmax))     (FP8)
//   q[k] = clamp(rint_half_even(fl32(x[k] / s)), -128, 127)             (INT8)
// the per-row scaled-FP8 formula of the TeleFuser "Quantization" page
// (section "Scaled FP8 checkpoints: W8A8"), with the reduced qmax of the
// LightX2V "模型量化技术" page (section "MiniMax-H3 FP8 FP16 累加"), and the
// symmetric INT8 formula of the TeleFuser page (section "Core ideas").
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "tfq_ptx.cuh"
#include "tfq_quant_common.cuh"

namespace tfq {
namespace {

// Two fp32 quotients t -> their INT8 codes rint_half_even(t) in bytes 0 and
// 1 (bytes 2 and 3 are don't-care).  Adding 1.5 * 2^23 rounds a |t| < 2^22
// to an integer, half to even, by the addition's own rounding, and leaves
// that integer in two's complement in the low bits of the sum.  No clamp to
// [-128, 127] is needed: with s = RN(amax / qmax), |x| <= amax and
// qmax <= 127, |t| <= RN(qmax * (1 + 2^-23)) < 127.5.
__device__ __forceinline__ uint32_t int8x2_rn(float2 t) {
    const float2 u = __fadd2_rn(t, make_float2(0x1.8p23f, 0x1.8p23f));
    return __byte_perm(__float_as_uint(u.x), __float_as_uint(u.y), 0x0040);
}

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
// quotient is below 2^-53 in magnitude, so only its sign reaches the codes
// (a = -0 may give +0 here; the caller restores the sign, see quantize8).
// Five packed fp32x2 instructions (sm_100: two IEEE round-to-nearest
// operations each, exactly the scalar ones) per pair of elements, no
// branch; nb = -b.  Kept as the reference form (TFQ_QUANT_DW_RCP=0); the
// quantizers use the four-instruction form below.  Both are checked against
// the IEEE division __fdiv_rn by tfq_selftest_div_rn.
__device__ __forceinline__ float2 div2_rn_from_rcp_unsigned_zero(float2 a, float2 nb, float2 y) {
    const float2 q0 = __fmul2_rn(a, y);
    const float2 r0 = __ffma2_rn(q0, nb, a);
    const float2 q1 = __ffma2_rn(r0, y, q0);
    const float2 r1 = __ffma2_rn(q1, nb, a);
    return __ffma2_rn(r1, y, q1);
}

// The same quotient in four packed instructions, from a two-term reciprocal
// y = RN(1/b), yl = RN((1 - b*y) * y) (1 - b*y is exact in one FMA and at
// most 2^-24 in magnitude, so y + yl is 1/b within 2^-47 relative).  Then
// q1 = RN(a*y + RN(a*yl)) is within half an ulp plus 2^-46 relative of a/b,
// hence faithful, and one Markstein step rounds it correctly.  Needs yl and
// a*yl normal, which holds for 2^-49 <= b <= 2^64 wherever |a/b| >= 2^-58
// (rows with a larger scale take the IEEE division; smaller quotients are
// below every code's rounding threshold and keep the sign of a, +0 for
// a = -0 as above).
__device__ __forceinline__ float2 div2_rn_from_rcp2_unsigned_zero(float2 a, float2 nb, float2 y, float2 yl) {
    const float2 q1 = __ffma2_rn(a, y, __fmul2_rn(a, yl));
    const float2 r = __ffma2_rn(q1, nb, a);
    return __ffma2_rn(r, y, q1);
}

#ifndef TFQ_QUANT_DW_RCP
#define TFQ_QUANT_DW_RCP 1  // 1: the four-instruction division from a two-term reciprocal
#endif

// Largest row scale the reciprocal-based division takes; larger ones use __fdiv_rn.
constexpr float kDivMaxScale = TFQ_QUANT_DW_RCP ? 0x1p64f : 0x1p125f;

// Low term of the row's reciprocal (0 when the five-instruction division is used).
__device__ __forceinline__ float rcp_low(float sc, float rcp) {
    return TFQ_QUANT_DW_RCP ? __fmul_rn(__fmaf_rn(-sc, rcp, 1.0f), rcp) : 0.0f;
}

// a / b for the quantizers (see the two functions above).
__device__ __forceinline__ float2 div2_rn_unsigned_zero(float2 a, float b, float y, float yl) {
#if TFQ_QUANT_DW_RCP
    return div2_rn_from_rcp2_unsigned_zero(a, make_float2(-b, -b), make_float2(y, y), make_float2(yl, yl));
#else
    (void)yl;
    return div2_rn_from_rcp_unsigned_zero(a, make_float2(-b, -b), make_float2(y, y));
#endif
}

// Quantizes the 8 bf16 values of `v` with scale `sc` (rcp = RN(1/sc)): 8
// output bytes.  kClamp: clamp x/s to +-qmax before the cast.  The clamp is
// skipped when qmax is an E4M3 value: then |x/s| <= qmax + 1 ulp(qmax)
// (s = RN(amax/qmax) and |x| <= amax), and qmax + 1 ulp encodes like qmax
// because the nearest E4M3 midpoint is 2^-4 of a binade away (448 + ulp
// saturates to 448).
// Two bf16 values (one 32-bit word) -> two codes in the low 16 bits (INT8:
// the high 16 bits are don't-care).
// (The Markstein quotient here may come out as +0 for a = -0; the caller
// restores the sign of zero codes from the inputs' sign bits, which is
// exact because every other quotient already carries the sign of a, and an
// INT8 code has no negative zero.)
template <bool kInt8, bool kClamp, bool kIeeeDiv>
__device__ __forceinline__ uint32_t quantize2(uint32_t w, float sc, float rcp, float rcp_lo, float qmax) {
    float a, b;
    if constexpr (kIeeeDiv) {
        a = __fdiv_rn(bf16_lo(w), sc);
        b = __fdiv_rn(bf16_hi(w), sc);
    } else {
        const float2 t = div2_rn_unsigned_zero(make_float2(bf16_lo(w), bf16_hi(w)), sc, rcp, rcp_lo);
        a = t.x;
        b = t.y;
    }
    if constexpr (kInt8) {
        return int8x2_rn(make_float2(a, b));
    } else {
        if constexpr (kClamp) {
            a = fminf(fmaxf(a, -qmax), qmax);
            b = fminf(fmaxf(b, -qmax), qmax);
        }
        return cvt_e4m3x2(a, b);
    }
}

template <bool kInt8, bool kClamp, bool kIeeeDiv>
__device__ __forceinline__ uint2 quantize8(uint4 v, float sc, float rcp, float rcp_lo, float qmax) {
    const uint32_t p0 = quantize2<kInt8, kClamp, kIeeeDiv>(v.x, sc, rcp, rcp_lo, qmax);
    const uint32_t p1 = quantize2<kInt8, kClamp, kIeeeDiv>(v.y, sc, rcp, rcp_lo, qmax);
    const uint32_t p2 = quantize2<kInt8, kClamp, kIeeeDiv>(v.z, sc, rcp, rcp_lo, qmax);
    const uint32_t p3 = quantize2<kInt8, kClamp, kIeeeDiv>(v.w, sc, rcp, rcp_lo, qmax);
    if constexpr (kInt8) return make_uint2(__byte_perm(p0, p1, 0x5410), __byte_perm(p2, p3, 0x5410));
    // E4M3 codes keep the sign of (negative) zero
    const uint32_t lo = p0 | (p1 << 16) | sign_bytes(v.x, v.y);
    const uint32_t hi = p2 | (p3 << 16) | sign_bytes(v.z, v.w);
    return make_uint2(lo, hi);
}

#ifndef TFQ_QUANT_L2_KEEP
#define TFQ_QUANT_L2_KEEP 1  // pass-1 loads ask L2 to keep the row for pass 2
#endif
// Load with an L2 cache policy (from createpolicy).
__device__ __forceinline__ uint4 ldg_nc_v4_policy(const uint4* p, uint64_t policy) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(policy));
    return v;
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

#ifndef TFQ_QUANT_SEG
#define TFQ_QUANT_SEG 16  // 16-byte units per lane per segment (a warp moves 32 * 16 * 16 B = 8 KiB)
#endif

template <bool kInt8, bool kClamp, bool kIeeeDiv, int SEG>
__device__ __forceinline__ void quantize_segment(const uint4 (&v)[SEG], uint2* qrow, int base, int lane, int units,
                                                 float sc, float rcp, float rcp_lo, float qmax) {
#pragma unroll
    for (int j = 0; j < SEG; ++j) {
        const int idx = base + lane + 32 * j;
        if (idx < units) qrow[idx] = quantize8<kInt8, kClamp, kIeeeDiv>(v[j], sc, rcp, rcp_lo, qmax);
    }
}

// Returns the row's L2 lines to normal eviction priority once pass 2 is done
// with them, so that the evict_last marks of pass 1 do not outlive the row
// and crowd the next kernel's working set out of L2.
__device__ __forceinline__ void release_row_l2(const uint4* row, int units, int lane) {
    const char* base = reinterpret_cast<const char*>(row);
    const int lines = (units * 16 + 127) / 128;
    for (int l = lane; l < lines; l += 32)
        asm volatile("applypriority.global.L2::evict_normal [%0], 128;" ::"l"(base + 128 * l) : "memory");
}

template <int SEG>
__device__ __forceinline__ void load_segment(uint4 (&v)[SEG], const uint4* row, int base, int lane, int units,
                                             uint64_t policy) {
#pragma unroll
    for (int j = 0; j < SEG; ++j) {
        const int idx = base + lane + 32 * j;
#if TFQ_QUANT_L2_KEEP
        v[j] = idx < units ? ldg_nc_v4_policy(row + idx, policy) : make_uint4(0u, 0u, 0u, 0u);
#else
        v[j] = idx < units ? ldg_nc_v4(row + idx) : make_uint4(0u, 0u, 0u, 0u);
#endif
    }
}

// One warp quantizes one row of `units` 16-byte units (K = 8 units) held at
// `row`: pass 1 loads a whole segment of SEG units per lane (a warp reads
// 512 contiguous bytes per load instruction) and reduces max |x| with packed
// max.xorsign.abs.bf16x2 and shuffles; pass 2 quantizes, from registers when
// the row fits one segment, else re-reading the row (from L2: pass 1 asked
// L2 to keep it).  Lane 0 writes the scale to *s_out; the codes go to qrow
// (8 per lane per store).  `keep` / `drop`: L2 policies for pass-1 loads of a
// row that is read again, and for loads read once.
template <bool kInt8, bool kClamp, int SEG>
__device__ __forceinline__ void quantize_row_warp(const uint4* row, int units, float qmax, uint2* qrow,
                                                  float* s_out, int lane, uint64_t keep, uint64_t drop) {
    const bool one_segment = units <= 32 * SEG;
    uint4 v[SEG];
    // pass 1: max |x|, a whole segment of loads in flight per warp
    uint32_t m = 0;
    for (int base = 0; base < units; base += 32 * SEG) {
        load_segment<SEG>(v, row, base, lane, units, one_segment ? drop : keep);
#pragma unroll
        for (int j = 0; j < SEG; ++j) m = max_abs4(m, v[j]);
    }
    m &= 0x7FFF7FFFu;
    float amax = fmaxf(bf16_lo(m), bf16_hi(m));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    const float sc = __fdiv_rn(fmaxf(amax, 1e-12f), qmax);
    const float rcp = __frcp_rn(sc);
    const float rcp_lo = rcp_low(sc, rcp);
    if (lane == 0) *s_out = sc;
    // pass 2: a row of one segment is still in registers; longer rows are
    // read again (from L2: the same row was read microseconds earlier)
    if (sc <= kDivMaxScale) {
        if (one_segment) {
            quantize_segment<kInt8, kClamp, false, SEG>(v, qrow, 0, lane, units, sc, rcp, rcp_lo, qmax);
        } else {
            for (int base = 0; base < units; base += 32 * SEG) {
                load_segment<SEG>(v, row, base, lane, units, drop);
                quantize_segment<kInt8, kClamp, false, SEG>(v, qrow, base, lane, units, sc, rcp, rcp_lo, qmax);
            }
        }
    } else {  // a huge scale: IEEE division (warp-uniform branch)
        for (int u = lane; u < units; u += 32)
            qrow[u] = quantize8<kInt8, kClamp, true>(ldg_nc_v4(row + u), sc, rcp, 0.0f, qmax);
    }
#if TFQ_QUANT_L2_KEEP
    if (!one_segment) release_row_l2(row, units, lane);
#endif
}

}  // namespace
}  // namespace tfq
