// tfq_quant_common.cuh -- bf16/E4M3 helpers shared by the row quantizers
// (tfq_quant.cu) and the MXFP8 block quantizer (tfq_quant_mx.cu).
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace tfq {
namespace {

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

// Sign bits of the four bf16 values in (w0, w1) moved to bit 7 of the four
// bytes of the result (the high byte of every bf16 carries its sign in bit 7).
__device__ __forceinline__ uint32_t sign_bytes(uint32_t w0, uint32_t w1) {
    return __byte_perm(w0, w1, 0x7531) & 0x80808080u;
}

// Global loads: 16 bytes, not allocated in L1.
__device__ __forceinline__ uint4 ldg_nc_v4(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Packed max of the magnitudes of the 8 bf16 values of v and the two in m.
__device__ __forceinline__ uint32_t max_abs4(uint32_t m, const uint4& v) {
    return max_abs_bf16x2(max_abs_bf16x2(m, v.x), max_abs_bf16x2(v.y, max_abs_bf16x2(v.z, v.w)));
}

}  // namespace
}  // namespace tfq
