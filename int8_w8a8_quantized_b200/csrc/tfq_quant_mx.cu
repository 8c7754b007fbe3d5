// tfq_quant_mx.cu -- MXFP8 block quantizer: BF16 -> E4M3FN codes with one
// E8M0 scale per 32 consecutive elements of a row, written in the
// scale-factor layout the block-scaled tensor-core MMA reads (include/tfq.h).
// The TeleFuser "Quantization" page (section "Offline conversion") names the
// format; the conversion is the one of the OCP Microscaling (MX) v1.0
// specification.  HBM-bandwidth bound.
#include <algorithm>

#include "tfq_internal.h"
#include "tfq_ptx.cuh"
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
#define TFQ_MX_CTAS 4  // resident CTAs of 8 warps per SM
#endif

// Byte of the scale-factor layout that holds the code of block b of row r
// (ra = 128-row panels): 512-byte atoms of 128 rows x 4 blocks, K-atom-major;
// row r owns word (r % 128) / 32 of line r % 32 of its atom.
__device__ __forceinline__ int64_t mx_sf_offset(int64_t r, int b, int64_t ra) {
    return ((static_cast<int64_t>(b >> 2) * ra + (r >> 7)) << 9) + ((r & 31) << 4) + (((r & 127) >> 5) << 2) + (b & 3);
}

// 16 bytes, read-only path, kept in L1: the four loads of a thread's 64-byte
// block come two per 32-byte sector, so the second of each pair hits L1.
__device__ __forceinline__ uint4 ldg_v4_l1(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

struct MxBlock {
    uint4 v[4];
};

__device__ __forceinline__ void mx_block_out(const MxBlock& k, int64_t g, int64_t r, int b, int nb, int ka4,
                                             int64_t ra, uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
    uint32_t m = max_abs_bf16x2(max_abs4(0u, k.v[0]), max_abs4(0u, k.v[1]));
    m = max_abs_bf16x2(m, max_abs_bf16x2(max_abs4(0u, k.v[2]), max_abs4(0u, k.v[3]))) & 0x7FFF7FFFu;
    const uint32_t code = e8m0_code(fmaxf(bf16_lo(m), bf16_hi(m)));
    const float inv = e8m0_inverse(code);
    const uint2 c0 = quantize8_mx(k.v[0], inv), c1 = quantize8_mx(k.v[1], inv);
    const uint2 c2 = quantize8_mx(k.v[2], inv), c3 = quantize8_mx(k.v[3], inv);
    uint4* dst = reinterpret_cast<uint4*>(q + g * 32);
    dst[0] = make_uint4(c0.x, c0.y, c1.x, c1.y);
    dst[1] = make_uint4(c2.x, c2.y, c3.x, c3.y);
    sf[mx_sf_offset(r, b, ra)] = static_cast<uint8_t>(code);
    if (b == nb - 1)  // the row's padding blocks up to a whole atom
        for (int p = nb; p < ka4; ++p) sf[mx_sf_offset(r, p, ra)] = 127;
}

// One thread per 32-value block: the matrix is a flat array of rows * K/32
// blocks of 64 bytes, thread t takes blocks t, t + S, t + 2S, ... (S = the
// grid's threads), two at a time (all eight 16-byte loads in flight).  The
// block maximum, its E8M0 code and reciprocal are computed once per block by
// one thread (no shuffles); consecutive threads read and write consecutive
// blocks (a warp's four loads cover 2 KB, its two 16-byte stores per thread
// 1 KB, each store instruction half of every 32-byte sector, which L2
// merges).  Padding scale entries (blocks past K / 32 up to a whole atom,
// rows past `rows` up to a whole 128-row panel) get code 127.  Measured on
// B200 against an atom-tiled kernel (a warp per 16 rows x 128 columns, four
// lanes per block, shuffles for the maximum and the codes): 1.1-1.2x alone,
// 4.45 -> 5.4 TB/s inside the video-DiT MXFP8 block (fewer instructions per
// element at the power-capped clock).
__global__ void __launch_bounds__(256, TFQ_MX_CTAS) quant_mxfp8_blocks_kernel(const uint4* __restrict__ x,
                                                                                    int64_t rows, int nb,
                                                                                    uint8_t* __restrict__ q,
                                                                                    uint8_t* __restrict__ sf) {
    pdl_allow_next();
    pdl_wait();
    const int64_t ra = (rows + 127) >> 7;
    const int ka4 = ((nb + 3) >> 2) << 2;
    const int64_t total = rows * nb;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t pad = (ra * 128 - rows) * ka4;
    for (int64_t i = tid; i < pad; i += stride) sf[mx_sf_offset(rows + i / ka4, static_cast<int>(i % ka4), ra)] = 127;
    // (row, block) of block g, advanced by `stride` blocks per step without a division
    const int64_t dr = stride / nb;
    const int db = static_cast<int>(stride - dr * nb);
    int64_t r = tid / nb;
    int b = static_cast<int>(tid - r * nb);
    for (int64_t g = tid; g < total; g += 2 * stride) {
        const int64_t g2 = g + stride;
        int64_t r2 = r + dr;
        int b2 = b + db;
        if (b2 >= nb) {
            b2 -= nb;
            ++r2;
        }
        MxBlock k1, k2;
#pragma unroll
        for (int j = 0; j < 4; ++j) k1.v[j] = ldg_v4_l1(x + g * 4 + j);
        if (g2 < total) {
#pragma unroll
            for (int j = 0; j < 4; ++j) k2.v[j] = ldg_v4_l1(x + g2 * 4 + j);
        }
        mx_block_out(k1, g, r, b, nb, ka4, ra, q, sf);
        if (g2 < total) mx_block_out(k2, g2, r2, b2, nb, ka4, ra, q, sf);
        r = r2 + dr;
        b = b2 + db;
        if (b >= nb) {
            b -= nb;
            ++r;
        }
    }
}

}  // namespace

tfq_status launch_quant_mxfp8(const void* x, int64_t rows, int64_t K, void* q, void* sf, cudaStream_t stream,
                              DeviceState* ds) {
    if (rows == 0 || K == 0) return TFQ_OK;
    // enough threads to take every block in one step of two, at most TFQ_MX_CTAS CTAs per SM
    const int64_t nblocks = rows * (K / 32);
    const int64_t grid = std::min<int64_t>((nblocks + 511) / 512, static_cast<int64_t>(ds->sm_count) * TFQ_MX_CTAS);
    const cudaError_t e = launch_kernel(quant_mxfp8_blocks_kernel, dim3(static_cast<unsigned>(std::max<int64_t>(grid, 1))),
                                        dim3(256), 0, stream, static_cast<const uint4*>(x), rows,
                                        static_cast<int>(K / 32), static_cast<uint8_t*>(q), static_cast<uint8_t*>(sf));
    return e == cudaSuccess ? TFQ_OK : fail(TFQ_ECUDA, "quantizer launch: %s", cudaGetErrorString(e));
}

}  // namespace tfq
