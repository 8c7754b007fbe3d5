// tfq_gemm_common.cuh -- pieces shared by the scaled GEMM kernels (tfq_gemm.cu)
// and the MXFP8 block-scaled kernels (tfq_gemm_mx.cu): tile constants, the
// kernel arguments, tile order and cluster pacing, L2 cache policies, and the
// epilogue that turns a finished TMEM accumulator into bf16 output tiles.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "tfq_internal.h"
#include "tfq_ptx.cuh"

namespace tfq {
namespace {

constexpr int BM = 128;            // tile rows (tokens)
constexpr int BN = 256;            // tile columns (output channels)
constexpr int BK = 128;            // K elements (= bytes) per stage: one 128-byte swizzle atom
constexpr int UMMA_K = 32;         // K per tcgen05.mma for 8-bit operands
constexpr int STAGES = 4;
constexpr int A_STAGE_BYTES = BM * BK;  // 16 KiB
constexpr int B_STAGE_BYTES = BN * BK;  // 32 KiB
constexpr int EPI_WARPS = 4;
constexpr int EPI_COLS = 64;                         // bf16 columns per TMA store (128 bytes)
constexpr int EPI_BUF_BYTES = 32 * EPI_COLS * 2;     // 4 KiB per staging buffer
constexpr int THREADS = 64 + EPI_WARPS * 32;         // producer warp, MMA warp, epilogue warps
constexpr int TMEM_COLS = 2 * BN;                    // double-buffered accumulator

constexpr size_t SMEM_RING = static_cast<size_t>(STAGES) * (A_STAGE_BYTES + B_STAGE_BYTES);
// Per epilogue warp: one output staging buffer and a copy of the tile's
// column scales and bias (fp32, 2 x BN floats).
constexpr size_t COLP_BYTES = 2 * BN * sizeof(float);
constexpr size_t SMEM_EPI = static_cast<size_t>(EPI_WARPS) * (EPI_BUF_BYTES + COLP_BYTES);
constexpr size_t SMEM_BARS = (2 * STAGES + 4 + 1) * 8 + 16;
constexpr size_t SMEM_BYTES = 1024 /* alignment slack */ + SMEM_RING + SMEM_EPI + SMEM_BARS;
static_assert(SMEM_BYTES <= 232448, "shared memory budget exceeded");

// Instruction descriptor of tcgen05.mma: accumulator format in bits 4-5
// (1 = F32 for kind::f8f6f4, 2 = S32 for kind::i8), A and B formats in bits
// 7-9 and 10-12 (E4M3 = 0 for f8f6f4; signed 8-bit = 1 for i8), both
// K-major (bits 15, 16 = 0), N >> 3 in bits 17-22, M >> 4 in bits 24-28.
// Accumulator kinds: F32 (E4M3 x E4M3, kind::f8f6f4), S32 (S8 x S8,
// kind::i8), F16 (E4M3 x E4M3 with a half-precision accumulator).
enum : int { kAccF32 = 0, kAccS32 = 1, kAccF16 = 2 };

template <int kAcc>
constexpr uint32_t make_idesc(int m, int n) {
    const uint32_t fmt = kAcc == kAccS32 ? (2u << 4) | (1u << 7) | (1u << 10)
                                         : (kAcc == kAccF16 ? 0u : (1u << 4));
    return fmt | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

// Linears that share their activations (and so the A operand) may run as one
// CTA-pair launch: at most this many.
constexpr int kMaxLinears = TFQ_MULTI_MAX_LINEARS;

struct GemmArgs {
    const float* s_a;
    const float* s_w;
    const uint16_t* bias;  // may be null
    int M, N, K;
    int m_tiles, n_tiles, k_blocks;
    // Tile order.  band_n > 0: bands of band_n consecutive N tiles; each band
    // sweeps every M tile (N fastest inside the band), so the band's weight
    // panels are reused by the whole sweep (kept in L2: evict_last) and the
    // activation panels stream (evict_first), re-read once per band.
    // band_n == 0: groups of group_m consecutive M tiles, each sweeping every
    // N tile (M fastest inside the group): activations kept, weights stream.
    int band_n;
    int group_m;
    uint32_t* err;
    // Cluster pacing (CTA-pair kernel): round_ctr[0] is zero when the launch
    // starts; the even CTA's producer adds 1 after issuing each tile's loads
    // and, before its round r, waits (up to TFQ_PACING_WAIT_NS, then goes on:
    // a performance hint, not a dependency) until every cluster has issued
    // its rounds before r.  Keeps the clusters within one tile of each other,
    // so the N tiles of a band that share an activation panel read it from L2
    // together instead of drifting apart and re-reading it from DRAM.
    // round_ctr[1] counts the clusters that are done; the last one sets both
    // words back to zero for the next launch given this slot (pacing_done),
    // so no memset sits between kernels in the stream, and a CUDA graph
    // replays the launch with the counter it expects.  Null: no pacing.
    unsigned* round_ctr;
    // CTA-pair kernel: when the last round has at most half as many tiles as
    // there are clusters, each of its tiles is split along N into two
    // half-width tiles (PBN / 2 columns, two clusters each), so that the
    // round takes about half a tile's time instead of a whole one.
    int tail_halves = 0;
    // The CTA-pair kernel that quantizes its own activations (null qx
    // otherwise): its quantizer warps turn bf16 rows of qx [M, K] into E4M3
    // codes qa [M, K] (the A operand its TMA loads read) and scales qs [M]
    // (= s_a), taking rows in increasing order from *q_next_row; each row
    // done adds one to q_share_rows[row / 128].  A CTA loads rows of A, and
    // reads their scales, only once their 128-row share is complete.
    const uint4* qx = nullptr;
    uint8_t* qa = nullptr;
    float* qs = nullptr;
    unsigned* q_next_row = nullptr;
    unsigned* q_share_rows = nullptr;
    float qmax = 0.0f;
    // The CTA-pair kernel: n_lin Linears that share A, their N tiles
    // concatenated (n_tiles counts them all); tile columns [lin_tile0[i],
    // lin_tile0[i + 1]) belong to Linear i, whose column scales, bias and N
    // are lin_s_w[i], lin_bias[i] and lin_N[i].  One Linear: lin_tile0 = {0,
    // n_tiles} and the three equal s_w, bias and N above.
    int n_lin = 1;
    int lin_tile0[kMaxLinears + 1] = {};
    const float* lin_s_w[kMaxLinears] = {};
    const uint16_t* lin_bias[kMaxLinears] = {};
    int lin_N[kMaxLinears] = {};
};

// The Linear a column of tiles belongs to, and the tile's column within it.
__device__ __forceinline__ void split_linear_tile(const GemmArgs& p, int tn_all, int& lin, int& tn) {
    lin = 0;
#pragma unroll
    for (int i = 1; i < kMaxLinears; ++i)
        if (i < p.n_lin && tn_all >= p.lin_tile0[i]) lin = i;
    tn = tn_all - p.lin_tile0[lin];
}

// The arguments of one tile's epilogue: those of its Linear.
__device__ __forceinline__ GemmArgs linear_args(const GemmArgs& p, int lin) {
    GemmArgs q = p;
    q.s_w = p.lin_s_w[lin];
    q.bias = p.lin_bias[lin];
    q.N = p.lin_N[lin];
    return q;
}

#ifndef TFQ_PACING_WAIT_NS
#define TFQ_PACING_WAIT_NS 200000ull
#endif

__device__ __forceinline__ void pace_round(const unsigned* ctr, int round, int total_tiles, int n_clusters) {
    if (ctr == nullptr || round < 1) return;
    const unsigned need = static_cast<unsigned>(min(total_tiles, round * n_clusters));
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 0; i < TFQ_WAIT_LIMIT_POLLS; ++i) {
        unsigned v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
        if (v >= need) return;
        if (globaltimer_ns() - t0 > TFQ_PACING_WAIT_NS) return;
    }
}

// Called once per cluster (the even CTA's producer thread) after its last
// round-counter update: counts the cluster as done; the last one of the
// launch sets the slot back to zero.  Every other cluster's round updates
// precede its own done count (the fence), so nothing adds to the counter
// after the reset.
__device__ __forceinline__ void pacing_done(unsigned* ctr, int n_clusters) {
    if (ctr == nullptr) return;
    __threadfence();
    if (atomicAdd(ctr + 1, 1u) == static_cast<unsigned>(n_clusters - 1)) {
        atomicExch(ctr, 0u);
        atomicExch(ctr + 1, 0u);
    }
}

__device__ __forceinline__ void tile_coords(int t, const GemmArgs& p, int& tm, int& tn) {
    if (p.band_n > 0) {
        const int per_band = p.band_n * p.m_tiles;
        const int bid = t / per_band;
        const int first_n = bid * p.band_n;
        const int gsize = min(p.n_tiles - first_n, p.band_n);
        const int r = t - bid * per_band;
        tn = first_n + r % gsize;
        tm = r / gsize;
        return;
    }
    const int per_group = p.group_m * p.n_tiles;
    const int gid = t / per_group;
    const int first_m = gid * p.group_m;
    const int gsize = min(p.m_tiles - first_m, p.group_m);
    const int r = t - gid * per_group;
    tm = first_m + r % gsize;
    tn = r / gsize;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// An accumulator word (one 32-bit TMEM column) as fp32: the F32 accumulator
// as is, the S32 one converted (round to nearest), the F16 one from the low
// half of its column.
template <int kAcc>
__device__ __forceinline__ float acc_value(uint32_t w) {
    if constexpr (kAcc == kAccS32) {
        return __int2float_rn(static_cast<int>(w));
    } else if constexpr (kAcc == kAccF16) {
        return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xFFFFu)));
    } else {
        return __uint_as_float(w);
    }
}

__device__ __forceinline__ void give_up(volatile int* abort_flag, uint32_t* err, uint32_t bit) {
    *abort_flag = 1;
    atomicOr(err, bit);
}

// Copies s_w[n] and bias[n] (as fp32; 0 past N or without bias) for the
// tile's kBN columns starting at n_tile0 into this warp's buffer colp
// (s_w at colp[0..kBN), bias at colp[kBN..2 kBN)).  Called while the MMA of
// the tile is still running, so the global-load latency is off the path.
// kUnitSw: the column scales are 1 (block-scaled GEMM, whose scales are
// applied by the tensor cores); s_w is not read.
template <int kBN, bool kUnitSw = false>
__device__ __forceinline__ void stage_col_params(const GemmArgs& p, float* colp, int n_tile0, int lane) {
    __syncwarp();  // the previous tile's reads of colp are done
    for (int g = lane; g < kBN / 8; g += 32) {
        const int n = n_tile0 + g * 8;
        float4 w0 = make_float4(0.f, 0.f, 0.f, 0.f), w1 = w0, b0 = w0, b1 = w0;
        if (n < p.N) {  // N % 8 == 0: a group of 8 columns is all valid or all out
            if constexpr (kUnitSw) {
                w0 = make_float4(1.f, 1.f, 1.f, 1.f);
                w1 = w0;
            } else {
                w0 = __ldg(reinterpret_cast<const float4*>(p.s_w + n));
                w1 = __ldg(reinterpret_cast<const float4*>(p.s_w + n + 4));
            }
            if (p.bias != nullptr) {
                const uint4 bv = __ldg(reinterpret_cast<const uint4*>(p.bias + n));
                b0 = make_float4(__uint_as_float(bv.x << 16), __uint_as_float(bv.x & 0xFFFF0000u),
                                 __uint_as_float(bv.y << 16), __uint_as_float(bv.y & 0xFFFF0000u));
                b1 = make_float4(__uint_as_float(bv.z << 16), __uint_as_float(bv.z & 0xFFFF0000u),
                                 __uint_as_float(bv.w << 16), __uint_as_float(bv.w & 0xFFFF0000u));
            }
        }
        float4* cw = reinterpret_cast<float4*>(colp + g * 8);
        float4* cb = reinterpret_cast<float4*>(colp + kBN + g * 8);
        cw[0] = w0;
        cw[1] = w1;
        cb[0] = b0;
        cb[1] = b1;
    }
    __syncwarp();
}

#ifndef TFQ_GEMM_POLICY_A
#define TFQ_GEMM_POLICY_A 0  // L2 policy of activation loads in N bands: 0 first, 1 normal, 2 last
#endif
#ifndef TFQ_GEMM_POLICY_B
#define TFQ_GEMM_POLICY_B 2  // L2 policy of weight loads in N bands: 0 first, 1 normal, 2 last
#endif

__device__ __forceinline__ uint64_t l2_policy(int kind) {
    return kind == 2 ? make_l2_policy_evict_last()
                     : (kind == 1 ? make_l2_policy_evict_normal() : make_l2_policy_evict_first());
}

// L2 policies of the operand loads: in N bands the band's weight panels are
// reused by the whole M sweep and are kept; the activation panels are reused
// only by the band's N tiles running at about the same time.  In M groups
// the roles swap.
__device__ __forceinline__ void l2_policies(const GemmArgs& p, uint64_t& pol_a, uint64_t& pol_b) {
    if (p.band_n > 0) {
        pol_a = l2_policy(TFQ_GEMM_POLICY_A);
        pol_b = l2_policy(TFQ_GEMM_POLICY_B);
    } else {
        pol_a = make_l2_policy_evict_last();
        pol_b = make_l2_policy_evict_normal();
    }
}

// Chunk c (EPI_COLS columns) of the epilogue of one 32-row slice of a
// finished tile; nothing past column N.  Its TMEM loads have completed when
// it returns, so the caller may hand those accumulator columns back.
template <int kBN, int kAcc>
__device__ __forceinline__ void store_tile_chunk(const GemmArgs& p, const CUtensorMap& tmY, uint32_t t_row,
                                                 uint8_t* ebuf, const float* colp, int n_tile0, int row0,
                                                 float2 sa2, uint64_t y_policy, int lane, int c) {
    const int n0 = n_tile0 + c * EPI_COLS;
    if (n0 >= p.N) return;  // uniform across the warp
    uint32_t acc[2][32];
    tmem_ld_32x32b_x32(t_row + c * EPI_COLS, acc[0]);
    tmem_ld_32x32b_x32(t_row + c * EPI_COLS + 32, acc[1]);
    tmem_ld_wait();
    uint32_t packed[2][16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {  // 8 columns
            const int nl = c * EPI_COLS + h * 32 + g * 8;
            const float4 w0 = *reinterpret_cast<const float4*>(colp + nl);
            const float4 w1 = *reinterpret_cast<const float4*>(colp + nl + 4);
            const float4 b0 = *reinterpret_cast<const float4*>(colp + kBN + nl);
            const float4 b1 = *reinterpret_cast<const float4*>(colp + kBN + nl + 4);
            const float2 sw[4] = {make_float2(w0.x, w0.y), make_float2(w0.z, w0.w), make_float2(w1.x, w1.y),
                                  make_float2(w1.z, w1.w)};
            const float2 bb[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w), make_float2(b1.x, b1.y),
                                  make_float2(b1.z, b1.w)};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 a2 = make_float2(acc_value<kAcc>(acc[h][g * 8 + 2 * j]),
                                              acc_value<kAcc>(acc[h][g * 8 + 2 * j + 1]));
                const float2 y = __ffma2_rn(__fmul2_rn(a2, sa2), sw[j], bb[j]);
                packed[h][g * 4 + j] = pack_bf16x2(y.x, y.y);
            }
        }
    }
    // The staging buffer's previous TMA store must have finished reading it.
    if (lane == 0) bulk_wait_read<0>();
    __syncwarp();
#pragma unroll
    for (int unit = 0; unit < 8; ++unit) {  // 128-byte swizzle: unit u of row r at u ^ (r % 8)
        uint4* dst = reinterpret_cast<uint4*>(ebuf + lane * 128 + ((unit ^ (lane & 7)) << 4));
        const uint32_t* w = &packed[unit >> 2][(unit & 3) * 4];
        *dst = make_uint4(w[0], w[1], w[2], w[3]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d_hint(&tmY, ebuf, n0, row0, y_policy);  // the output streams out of L2
        bulk_commit();
    }
}

// Epilogue of one 32-row slice of a finished tile: TMEM -> registers ->
// y = acc * s_a[m] * s_w[n] + bias[n] in fp32 (packed fp32x2 operations) ->
// bf16 -> 128-byte swizzled staging buffer -> TMA store, EPI_COLS columns
// at a time (store_tile_chunk).  `t_row` is the TMEM address of this warp's
// 32 lanes at the tile's first column; colp holds the tile's column scales
// and bias.
// `ncols` (a multiple of EPI_COLS, at most kBN): columns of the tile to store.
template <int kBN, int kAcc>
__device__ __forceinline__ void store_tile_rows(const GemmArgs& p, const CUtensorMap& tmY, uint32_t t_row,
                                                uint8_t* ebuf, const float* colp, int n_tile0, int row0, float sa,
                                                int lane, int ncols = kBN) {
    const float2 sa2 = make_float2(sa, sa);
    const uint64_t y_policy = make_l2_policy_evict_first();
#pragma unroll 1
    for (int c = 0; c < ncols / EPI_COLS; ++c)
        store_tile_chunk<kBN, kAcc>(p, tmY, t_row, ebuf, colp, n_tile0, row0, sa2, y_policy, lane, c);
}

__device__ __forceinline__ void pair_tile_coords(int t, int m_tiles, int n_tiles, int group_m, int band_n, int& tm,
                                                 int& tn) {
    if (band_n > 0) {
        const int per_band = band_n * m_tiles;
        const int bid = t / per_band;
        const int first_n = bid * band_n;
        const int gsize = min(n_tiles - first_n, band_n);
        const int r = t - bid * per_band;
        tn = first_n + r % gsize;
        tm = r / gsize;
        return;
    }
    const int per_group = group_m * n_tiles;
    const int gid = t / per_group;
    const int first_m = gid * group_m;
    const int gsize = min(m_tiles - first_m, group_m);
    const int r = t - gid * per_group;
    tm = first_m + r % gsize;
    tn = r / gsize;
}

// Work item w of a cluster of the CTA-pair kernel (w = cluster, cluster +
// n_clusters, ...): tile t whole (half = -1) or, in a split last round
// (GemmArgs::tail_halves), half `half` (0: first PBN / 2 columns, 1: the
// rest) of tile t.  Returns false past the last item.
__device__ __forceinline__ bool pair_work_item(int w, int total_tiles, int n_clusters, int tail_halves, int& t,
                                               int& half) {
    const int whole = tail_halves ? (total_tiles / n_clusters) * n_clusters : total_tiles;
    if (w < whole) {
        t = w;
        half = -1;
        return true;
    }
    const int j = w - whole;
    if (!tail_halves || j >= 2 * (total_tiles - whole)) return false;
    t = whole + (j >> 1);
    half = j & 1;
    return true;
}

// Host side: split the last round when it holds at most n_clusters / 2 tiles.
inline int choose_tail_halves(int64_t total_tiles, int64_t n_clusters) {
#ifdef TFQ_GEMM_NO_TAIL_HALVES
    return 0;
#else
    const int64_t last = total_tiles % n_clusters;
    return (last > 0 && 2 * last <= n_clusters) ? 1 : 0;
#endif
}

#ifndef TFQ_GEMM_PAIR_MIN_M
#define TFQ_GEMM_PAIR_MIN_M 512  // below this many rows the 1-CTA 128 x 256 tiles are used
#endif

bool use_pair_kernel(int64_t M, int sm_count) { return M >= TFQ_GEMM_PAIR_MIN_M && sm_count >= 2; }

#ifndef TFQ_GEMM_BAND_MB
#define TFQ_GEMM_BAND_MB 40     // > 0: N bands holding about this many MB of weight; 0: M groups
#endif
#ifndef TFQ_GEMM_GROUP_M
#define TFQ_GEMM_GROUP_M 8
#endif

// Raster order (see GemmArgs): N bands whose weight panels total about
// TFQ_GEMM_BAND_MB, or M groups of TFQ_GEMM_GROUP_M tiles.
void choose_raster(int64_t K, int bn, int& band_n, int& group_m) {
    group_m = TFQ_GEMM_GROUP_M;
    band_n = 0;
    if (TFQ_GEMM_BAND_MB > 0) {
        const int64_t panel = static_cast<int64_t>(bn) * K;  // bytes of one N tile's weight panel
        band_n = static_cast<int>(std::max<int64_t>(1, static_cast<int64_t>(TFQ_GEMM_BAND_MB) * 1000000 / panel));
    }
}

}  // namespace
}  // namespace tfq
