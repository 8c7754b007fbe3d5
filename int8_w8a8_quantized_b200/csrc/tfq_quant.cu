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
// Design (B200): rows of K <= 2048 go to a grouped kernel: a power-of-two
// group of lanes per row, several rows per warp, each lane holding 1, 4 or 8
// of the row's 16-byte units, so that a warp keeps kilobytes in flight
// however short the row.  Longer rows: one warp per row, rows strided over a grid of two or three
// CTAs of eight warps per SM (rows of 16384 <= K <= 32768 are staged in
// shared memory instead, see below).  Pass 1 loads a whole segment of the
// row (12, 16 or 20 16-byte loads per lane: 6-10 KiB per warp in flight, a
// warp reads 512 contiguous bytes per load) and reduces |x| with packed
// max.xorsign.abs.bf16x2 and shuffles.  Pass 2 quantizes: a row of at most
// one segment is still in registers; a longer row is
// read again, which hits L2 because pass 1 loaded it with an evict_last
// cache policy (so HBM sees 2 bytes read and 1 written per element).  The
// division is a branch-free correctly rounded one (a two-term reciprocal of
// the row scale and one Markstein correction, four packed instructions per
// pair of values); two values are converted per cvt instruction and a lane
// stores 8 codes at a time (a warp writes 256 contiguous bytes).
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>

#include "tfq_internal.h"
#include "tfq_ptx.cuh"
#include "tfq_quant_common.cuh"
#include "tfq_quant_row.cuh"

namespace tfq {
namespace {

constexpr int kCtasPerSm = 2;  // 8 warps per CTA; ~125 registers per thread allow two per SM

#ifndef TFQ_QUANT_SHORT_SEG
#define TFQ_QUANT_SHORT_SEG 12  // segment of the variant for rows of K <= 32 * 12 * 8 = 3072
#endif
#ifndef TFQ_QUANT_WIDE_SEG
#define TFQ_QUANT_WIDE_SEG 20   // segment of the variant that holds a K = 5120 row in one pass
#endif
#ifndef TFQ_QUANT_SHORT_SEG_MAX_ROWS
#define TFQ_QUANT_SHORT_SEG_MAX_ROWS 32768  // ... used for at most this many rows
#endif

// Resident CTAs per SM of the warp-per-row kernel for a segment size: the
// short-segment variant holds fewer registers, so three CTAs fit.
template <int SEG>
constexpr int rows_ctas_per_sm() {
    return SEG <= TFQ_QUANT_SHORT_SEG ? 3 : kCtasPerSm;
}

template <bool kInt8, bool kClamp, int SEG>
__global__ void __launch_bounds__(256, rows_ctas_per_sm<SEG>()) quant_rows_kernel(const uint4* __restrict__ x,
                                                                                 int64_t M, int K, float qmax,
                                                                                 uint8_t* __restrict__ q,
                                                                                 float* __restrict__ s) {
    pdl_allow_next();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int units = K >> 3;  // 16-byte units of 8 bf16 per row
    const uint64_t keep = l2_policy_evict_last(), drop = l2_policy_evict_first();
    for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < M; r += nwarps)
        quantize_row_warp<kInt8, kClamp, SEG>(x + r * units, units, qmax, reinterpret_cast<uint2*>(q + r * K),
                                              s + r, lane, keep, drop);
}

// Rows of 16384 <= K <= TFQ_QUANT_STAGED_MAX_K: the row is staged in shared
// memory.  (Measured on B200: below K = 16384 the one-warp-per-row loop above
// is as fast or faster inside the DiT block -- staging its K = 13824
// activation made the block's quantizers 6 % slower, though that row length
// ran 10 % faster alone -- while for K >= 16384 staging is 20 to 35 % faster
// alone.)  A CTA of
// 256 threads quantizes one row at a time while the TMA
// engine brings its next rows (one bulk copy of a whole row into each of 2 to
// 4 row buffers, completion counted on that buffer's mbarrier).  Pass 1
// reduces max |x| over the buffer (warp shuffles, then the 8 warp maxima
// through shared memory), pass 2 quantizes from the same buffer.  HBM sees the
// row read once and L2 carries it once; the one-warp-per-row loop above reads
// rows longer than one segment twice from L2.
#ifndef TFQ_QUANT_STAGED_MAX_K
#define TFQ_QUANT_STAGED_MAX_K 32768  // two row buffers of 2 K bytes: 128 KiB at this K
#endif
#ifndef TFQ_QUANT_STAGED_MIN_K
#define TFQ_QUANT_STAGED_MIN_K 16384  // shorter rows: grouped kernel or one warp per row
#endif
constexpr int kStagedThreads = 256;
constexpr int kStagedMaxSlots = 4;
constexpr int kStagedSmemLimit = 200 * 1024;
#ifndef TFQ_QUANT_STAGED_SLOT_BYTES
#define TFQ_QUANT_STAGED_SLOT_BYTES (96 * 1024)  // row buffers per CTA: as many as fit here, 2 to 4
#endif

template <bool kInt8, bool kClamp>
__global__ void __launch_bounds__(kStagedThreads) quant_rows_staged_kernel(const uint4* __restrict__ x, int64_t M,
                                                                           int K, int slots, float qmax,
                                                                           uint8_t* __restrict__ q,
                                                                           float* __restrict__ s, uint32_t* err) {
    pdl_allow_next();
    pdl_wait();
    extern __shared__ __align__(128) uint8_t staged_smem[];
    __shared__ uint64_t bar[kStagedMaxSlots];
    __shared__ float wmax[kStagedThreads / 32];
    __shared__ int abort_flag;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int units = K >> 3;
    const uint32_t row_bytes = static_cast<uint32_t>(K) * 2u;
    const int64_t stride = gridDim.x;
    if (tid == 0) {
        for (int i = 0; i < slots; ++i) mbar_init(&bar[i], 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        for (int i = 0; i < slots; ++i) {
            const int64_t r = blockIdx.x + i * stride;
            if (r < M) {
                mbar_arrive_expect_tx(&bar[i], row_bytes);
                bulk_g2s(staged_smem + static_cast<size_t>(i) * row_bytes, x + r * units, row_bytes, &bar[i]);
            }
        }
    }
    int it = 0;
    for (int64_t r = blockIdx.x; r < M; r += stride, ++it) {
        const int sl = it % slots;
        const uint32_t ph = static_cast<uint32_t>(it / slots) & 1u;
        if (tid == 0 && !mbar_wait(&bar[sl], ph, &abort_flag)) {
            abort_flag = 1;
            atomicOr(err, kErrQuantStage);
        }
        __syncthreads();
        if (abort_flag) break;
        (void)mbar_try_wait(&bar[sl], ph);  // completed: makes the copied row visible to this thread
        const uint4* row = reinterpret_cast<const uint4*>(staged_smem + static_cast<size_t>(sl) * row_bytes);
        uint32_t m = 0;
        for (int u = tid; u < units; u += kStagedThreads) m = max_abs4(m, row[u]);
        m &= 0x7FFF7FFFu;
        float amax = fmaxf(bf16_lo(m), bf16_hi(m));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        if (lane == 0) wmax[warp] = amax;
        __syncthreads();
        amax = wmax[0];
#pragma unroll
        for (int w = 1; w < kStagedThreads / 32; ++w) amax = fmaxf(amax, wmax[w]);
        const float sc = __fdiv_rn(fmaxf(amax, 1e-12f), qmax);
        if (tid == 0) s[r] = sc;
        uint2* qrow = reinterpret_cast<uint2*>(q + r * K);
        if (sc <= kDivMaxScale) {
            const float rcp = __frcp_rn(sc);
            const float rcp_lo = rcp_low(sc, rcp);
            for (int u = tid; u < units; u += kStagedThreads)
                qrow[u] = quantize8<kInt8, kClamp, false>(row[u], sc, rcp, rcp_lo, qmax);
        } else {  // a huge scale: IEEE division (uniform across the CTA)
            for (int u = tid; u < units; u += kStagedThreads)
                qrow[u] = quantize8<kInt8, kClamp, true>(row[u], sc, 0.0f, 0.0f, qmax);
        }
        __syncthreads();  // every thread is done with this buffer and with wmax
        if (tid == 0) {
            const int64_t rn = r + slots * stride;
            if (rn < M) {
                mbar_arrive_expect_tx(&bar[sl], row_bytes);
                bulk_g2s(staged_smem + static_cast<size_t>(sl) * row_bytes, x + rn * units, row_bytes, &bar[sl]);
            }
        }
    }
    // After giving up, the copies still in flight must land (bounded) before
    // this CTA's shared memory is released.
    if (abort_flag && tid == 0) {
        for (int k = 0; k < slots; ++k) {
            const int j = it + k;
            if (blockIdx.x + static_cast<int64_t>(j) * stride < M)
                (void)mbar_wait(&bar[j % slots], static_cast<uint32_t>(j / slots) & 1u, nullptr);
        }
    }
}

#ifndef TFQ_QUANT_J4_CTAS
#define TFQ_QUANT_J4_CTAS 4  // resident CTAs of 8 warps per SM for the grouped kernel with 4 units per lane
#endif
#ifndef TFQ_QUANT_J8_CTAS
#define TFQ_QUANT_J8_CTAS 3  // ... with 8 units per lane (~70 registers)
#endif
#ifndef TFQ_QUANT_FORCE_J
#define TFQ_QUANT_FORCE_J 0  // 0: choose units per lane from the row length (1, 4 or 8 to force one)
#endif
constexpr int kGroupMaxUnits = 256;  // rows of K <= 2048 take the grouped kernel

template <int J>
constexpr int grouped_ctas_per_sm() {
    return J == 1 ? 8 : J == 4 ? TFQ_QUANT_J4_CTAS : TFQ_QUANT_J8_CTAS;
}

// Short and mid-length rows (K <= 2048: a head_dim vector of a KV cache, the
// hidden size of a small DiT): LPR lanes share a row, so a warp holds 32 / LPR
// rows at a time; lane `sub` of a row holds its 16-byte units sub, sub + LPR,
// sub + 2 LPR, ... (at most J of them).  Each load instruction then reads LPR
// consecutive units of every row in the warp, all of a row's loads are in
// flight together, and the max reduction stays inside each LPR-lane group.
// A one-row-per-warp loop would keep only K * 2 bytes per warp in flight,
// too little to cover HBM latency for K of a few hundred.
template <bool kInt8, bool kClamp, int LPR, int J>
__global__ void __launch_bounds__(256, grouped_ctas_per_sm<J>()) quant_grouped_rows_kernel(const uint4* __restrict__ x, int64_t M, int K,
                                                                 float qmax, uint8_t* __restrict__ q,
                                                                 float* __restrict__ s) {
    pdl_allow_next();
    pdl_wait();
    constexpr int RPW = 32 / LPR;  // rows per warp
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPR;
    const int units = K >> 3;      // <= LPR * J
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t base = warp * RPW; base < M; base += nwarps * RPW) {
        const int64_t r = base + lane / LPR;
        const bool row_ok = r < M;
        uint4 v[J];
        uint32_t m = 0;
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int u = sub + LPR * j;
            v[j] = (row_ok && u < units) ? ldg_nc_v4(x + r * units + u) : make_uint4(0u, 0u, 0u, 0u);
            m = max_abs4(m, v[j]);
        }
        m &= 0x7FFF7FFFu;
        float amax = fmaxf(bf16_lo(m), bf16_hi(m));
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        const float sc = __fdiv_rn(fmaxf(amax, 1e-12f), qmax);
        if (row_ok) {
            if (sub == 0) s[r] = sc;
            uint2* qrow = reinterpret_cast<uint2*>(q + r * K);
            if (sc <= kDivMaxScale) {
                const float rcp = __frcp_rn(sc);
                const float rcp_lo = rcp_low(sc, rcp);
#pragma unroll
                for (int j = 0; j < J; ++j) {
                    const int u = sub + LPR * j;
                    if (u < units) qrow[u] = quantize8<kInt8, kClamp, false>(v[j], sc, rcp, rcp_lo, qmax);
                }
            } else {  // a huge scale: IEEE division for this row
#pragma unroll
                for (int j = 0; j < J; ++j) {
                    const int u = sub + LPR * j;
                    if (u < units) qrow[u] = quantize8<kInt8, kClamp, true>(v[j], sc, 0.0f, 0.0f, qmax);
                }
            }
        }
    }
}

// Element-wise self-check of div_rn_from_rcp against the IEEE division.
__global__ void div_selftest_kernel(const float* __restrict__ a, const float* __restrict__ b, int64_t n,
                                    float* __restrict__ ours, float* __restrict__ ieee) {
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float x = a[i], y = b[i];
        const float r = __frcp_rn(y);
        // the packed form the quantizers use; both lanes carry the same
        // quotient, the sign of a zero result is restored as the quantizers do
        const float2 t = div2_rn_unsigned_zero(make_float2(x, x), y, r, rcp_low(y, r));
        ours[i] = copysignf(t.y, x);
        ieee[i] = __fdiv_rn(x, y);
    }
}

// K == 0: an empty row has amax 0, so only the floored scale is written.
__global__ void empty_rows_scale_kernel(int64_t M, float qmax, float* s) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < M) s[i] = __fdiv_rn(1e-12f, qmax);
}


template <int LPR, int J>
void launch_grouped_lpr(const void* x, int64_t rows, int64_t K, float qmax, bool out_int8, bool clamp, void* q,
                        float* s, cudaStream_t stream, int64_t blocks) {
    auto kernel = out_int8 ? quant_grouped_rows_kernel<true, false, LPR, J>
                           : (clamp ? quant_grouped_rows_kernel<false, true, LPR, J>
                                    : quant_grouped_rows_kernel<false, false, LPR, J>);
    // a launch error is also the runtime's last error, which the caller reads
    (void)launch_kernel(kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream, static_cast<const uint4*>(x),
                        rows, static_cast<int>(K), qmax, static_cast<uint8_t*>(q), s);
}

template <int J>
void launch_grouped_j(int lpr, const void* x, int64_t rows, int64_t K, float qmax, bool out_int8, bool clamp,
                      void* q, float* s, cudaStream_t stream, int sm_count) {
    const int64_t rows_per_block = 8 * (32 / lpr);
    const int64_t blocks = std::min<int64_t>((rows + rows_per_block - 1) / rows_per_block,
                                             static_cast<int64_t>(sm_count) * grouped_ctas_per_sm<J>());
    switch (lpr) {
        case 2: launch_grouped_lpr<2, J>(x, rows, K, qmax, out_int8, clamp, q, s, stream, blocks); break;
        case 4: launch_grouped_lpr<4, J>(x, rows, K, qmax, out_int8, clamp, q, s, stream, blocks); break;
        case 8: launch_grouped_lpr<8, J>(x, rows, K, qmax, out_int8, clamp, q, s, stream, blocks); break;
        case 16: launch_grouped_lpr<16, J>(x, rows, K, qmax, out_int8, clamp, q, s, stream, blocks); break;
        default: launch_grouped_lpr<32, J>(x, rows, K, qmax, out_int8, clamp, q, s, stream, blocks); break;
    }
}

struct GroupShape {
    int lpr;    // lanes per row (a power of two, 2..32)
    int j;      // units per lane (1, 4 or 8)
    int waste;  // lane slots left empty per row: lpr * j - units
};

GroupShape group_shape(int units, int j) {
    int lpr = 2;
    while (lpr * j < units) lpr *= 2;
    return {lpr, j, lpr * j - units};
}

// Lanes per row and units per lane for a row of `units` 16-byte units
// (units <= kGroupMaxUnits), from a sweep of K = 16..2048 on B200 (1 GiB of
// input per call): 4 units per lane wins where it fills every lane slot
// (K = 64, 128, 256, 512, 1024) and where 8 units per lane would leave only
// two lanes per row; otherwise the shape with fewer empty slots, 8 units per
// lane on a tie; one unit per lane for rows of K <= 16.
GroupShape pick_group_shape(int units) {
    if (TFQ_QUANT_FORCE_J != 0) return group_shape(units, TFQ_QUANT_FORCE_J);
    if (units <= 2) return group_shape(units, 1);
    const GroupShape g8 = group_shape(units, 8);
    if (units > 128) return g8;
    const GroupShape g4 = group_shape(units, 4);
    if (g4.waste == 0 || g8.lpr == 2) return g4;
    return g4.waste < g8.waste ? g4 : g8;
}

tfq_status launch_grouped_rows(const void* x, int64_t rows, int64_t K, float qmax, bool out_int8, bool clamp,
                               void* q, float* s, cudaStream_t stream, DeviceState* ds) {
    const GroupShape g = pick_group_shape(static_cast<int>(K / 8));
    if (g.lpr > 32) return fail(TFQ_EUNSUPPORTED, "row of K=%lld does not fit one warp", (long long)K);
    switch (g.j) {
        case 1: launch_grouped_j<1>(g.lpr, x, rows, K, qmax, out_int8, clamp, q, s, stream, ds->sm_count); break;
        case 4: launch_grouped_j<4>(g.lpr, x, rows, K, qmax, out_int8, clamp, q, s, stream, ds->sm_count); break;
        default: launch_grouped_j<8>(g.lpr, x, rows, K, qmax, out_int8, clamp, q, s, stream, ds->sm_count); break;
    }
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TFQ_OK : fail(TFQ_ECUDA, "quantizer launch: %s", cudaGetErrorString(e));
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

namespace {

tfq_status launch_staged_rows(const void* x, int64_t rows, int64_t K, float qmax, bool out_int8, bool clamp, void* q,
                              float* s, cudaStream_t stream, DeviceState* ds) {
    auto kernel = out_int8 ? quant_rows_staged_kernel<true, false>
                           : (clamp ? quant_rows_staged_kernel<false, true> : quant_rows_staged_kernel<false, false>);
    if (!ds->quant_attr_set) {
        const void* fns[3] = {reinterpret_cast<const void*>(quant_rows_staged_kernel<true, false>),
                              reinterpret_cast<const void*>(quant_rows_staged_kernel<false, true>),
                              reinterpret_cast<const void*>(quant_rows_staged_kernel<false, false>)};
        for (const void* f : fns) {
            const cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kStagedSmemLimit);
            if (e != cudaSuccess) return fail(TFQ_ECUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        }
        ds->quant_attr_set = true;
    }
    const int slots = static_cast<int>(std::min<int64_t>(
        kStagedMaxSlots, std::max<int64_t>(2, TFQ_QUANT_STAGED_SLOT_BYTES / (2 * K))));
    const size_t smem = static_cast<size_t>(slots) * 2 * static_cast<size_t>(K);
    int per_sm = 0;
    const cudaError_t eo = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kStagedThreads, smem);
    if (eo != cudaSuccess || per_sm < 1) return fail(TFQ_ECUDA, "staged quantizer occupancy: %s", cudaGetErrorString(eo));
    const int64_t blocks = std::min<int64_t>(rows, static_cast<int64_t>(ds->sm_count) * per_sm);
    const cudaError_t e = launch_kernel(kernel, dim3(static_cast<unsigned>(blocks)), dim3(kStagedThreads), smem,
                                        stream, static_cast<const uint4*>(x), rows, static_cast<int>(K), slots, qmax,
                                        static_cast<uint8_t*>(q), s, ds->err_word);
    return e == cudaSuccess ? TFQ_OK : fail(TFQ_ECUDA, "quantizer launch: %s", cudaGetErrorString(e));
}

}  // namespace

bool is_e4m3_value(float v) {
    int e = 0;
    const float m = std::frexp(v, &e) * 16.0f;  // 4 significant bits -> integer
    return v >= 0x1p-6f && v <= 448.0f && m == std::floor(m);
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
    const bool clamp = !out_int8 && !is_e4m3_value(qmax);
    if (K / 8 <= kGroupMaxUnits) return launch_grouped_rows(x, rows, K, qmax, out_int8, clamp, q, s, stream, ds);
    if (K >= TFQ_QUANT_STAGED_MIN_K && K <= TFQ_QUANT_STAGED_MAX_K)
        return launch_staged_rows(x, rows, K, qmax, out_int8, clamp, q, s, stream, ds);
    constexpr int kLong = TFQ_QUANT_SEG, kWide = TFQ_QUANT_WIDE_SEG, kShort = TFQ_QUANT_SHORT_SEG;
    // Few rows (each warp gets only a handful): the variant with three CTAs per
    // SM hides more latency -- [8192, 3072] 4.2 vs 3.8 TB/s; many rows: the
    // two-CTA one is faster ([174762, 3072] 6.3 vs 5.7 TB/s), measured on B200.
    const bool short_seg = K <= 32 * kShort * 8 && rows <= TFQ_QUANT_SHORT_SEG_MAX_ROWS;
    // Otherwise the segment (16 or 20 units per lane) that leaves fewer lane
    // slots of the last segment empty: K = 5120 fits one 20-unit segment (a
    // single pass, no re-read from L2), K = 13824 three instead of four; 16 on
    // a tie.  Measured on B200 inside the video-DiT block: 4.7-4.9 vs 4.0 TB/s.
    const int64_t units = K / 8;
    auto waste = [&](int seg) { return (units + 32 * seg - 1) / (32 * seg) * (32 * seg) - units; };
    const bool wide = !short_seg && waste(kWide) < waste(kLong);
    const int variant = out_int8 ? 0 : (clamp ? 1 : 2);
    using Kernel = void (*)(const uint4*, int64_t, int, float, uint8_t*, float*);
    const Kernel short_k[3] = {quant_rows_kernel<true, false, kShort>, quant_rows_kernel<false, true, kShort>,
                               quant_rows_kernel<false, false, kShort>};
    const Kernel wide_k[3] = {quant_rows_kernel<true, false, kWide>, quant_rows_kernel<false, true, kWide>,
                              quant_rows_kernel<false, false, kWide>};
    const Kernel long_k[3] = {quant_rows_kernel<true, false, kLong>, quant_rows_kernel<false, true, kLong>,
                              quant_rows_kernel<false, false, kLong>};
    const Kernel kernel = short_seg ? short_k[variant] : (wide ? wide_k[variant] : long_k[variant]);
    const int threads = 256;  // 8 warps, one row per warp at a time
    const int ctas_per_sm = short_seg ? rows_ctas_per_sm<kShort>()
                                      : (wide ? rows_ctas_per_sm<kWide>() : rows_ctas_per_sm<kLong>());
    const int64_t blocks = std::min<int64_t>((rows + 7) / 8, static_cast<int64_t>(ds->sm_count) * ctas_per_sm);
    const cudaError_t e = launch_kernel(kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, stream,
                                        static_cast<const uint4*>(x), rows, static_cast<int>(K), qmax,
                                        static_cast<uint8_t*>(q), s);
    return e == cudaSuccess ? TFQ_OK : fail(TFQ_ECUDA, "quantizer launch: %s", cudaGetErrorString(e));
}

}  // namespace tfq
