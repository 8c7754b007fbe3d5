// tfq_gemm.cu -- scaled FP8 GEMM with fused epilogue on 5th-generation
// tensor cores (tcgen05, sm_100a).
//
// Computes out[m,n] = bf16_rn(acc[m,n] * s_a[m] * s_w[n] + bias[n]) with
// acc[m,n] = sum_k e4m3(A[m,k]) * e4m3(W[n,k]) accumulated in fp32: the
// scaled GEMM of the TeleFuser "Quantization" page (sections "Scaled FP8
// checkpoints" and "tf-kernel FP8: online W8A8": per-token activation
// scales, per-output-channel weight scales, BF16 output).
//
// Kernel structure (one persistent CTA per SM, 192 threads):
//   warp 0      TMA producer: streams 128x128 A tiles and 256x128 B tiles
//               (K-major, 128-byte swizzle) into a 4-stage shared-memory
//               ring, completion counted on "full" mbarriers.
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators)
//               and, from one thread, issues tcgen05.mma kind::f8f6f4
//               (M=128, N=256, K=32 per instruction, 4 per stage); each
//               stage is released to the producer by tcgen05.commit onto its
//               "empty" mbarrier, each finished tile by a commit onto the
//               accumulator's "tmem_full" mbarrier.
//   warps 2..5  epilogue: tcgen05.ld a 32-row quarter of the accumulator
//               (warp w may read TMEM lanes 32*(w%4)..+31), apply s_a, s_w
//               and bias in fp32, round to bf16, write 64-column chunks into
//               a 128-byte-swizzled staging buffer and TMA-store them; the
//               accumulator is handed back through "tmem_empty" so the MMA
//               of the next tile overlaps this epilogue.
// Tiles are visited in M-grouped raster order so that the CTAs running at
// the same time share A and B panels in L2.  M and N tails are handled by
// TMA (zero fill on load, clipping on store); K tails by zero fill.
// Every wait is bounded (see tfq_ptx.cuh); a CTA that gives up records it in
// the error word, drains its own outstanding copies and MMAs, frees TMEM and
// returns.
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
    // Cluster pacing (CTA-pair kernel): zeroed before the launch; the even
    // CTA's producer adds 1 after issuing each tile's loads and, before its
    // round r, waits (up to TFQ_PACING_WAIT_NS, then goes on: a performance
    // hint, not a dependency) until every cluster has issued its rounds
    // before r.  Keeps the clusters within one tile of each other, so the N
    // tiles of a band that share an activation panel read it from L2 together
    // instead of drifting apart and re-reading it from DRAM.  Null: no pacing.
    unsigned* round_ctr;
};

#ifndef TFQ_PACING_WAIT_NS
#define TFQ_PACING_WAIT_NS 200000ull
#endif

__device__ __forceinline__ void pace_round(const unsigned* ctr, int round, int total_tiles, int n_clusters) {
    if (ctr == nullptr || round < 1) return;
    const long long need = min(static_cast<long long>(total_tiles), static_cast<long long>(round) * n_clusters);
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 0; i < TFQ_WAIT_LIMIT_POLLS; ++i) {
        unsigned v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
        if (static_cast<long long>(v) >= need) return;
        if (globaltimer_ns() - t0 > TFQ_PACING_WAIT_NS) return;
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

// Epilogue of one 32-row slice of a finished tile: TMEM -> registers ->
// y = acc * s_a[m] * s_w[n] + bias[n] in fp32 (packed fp32x2 operations) ->
// bf16 -> 128-byte swizzled staging buffer -> TMA store, EPI_COLS columns
// at a time.  `t_row` is the TMEM address of this warp's 32 lanes at the
// tile's first column; colp holds the tile's column scales and bias.
template <int kBN, int kAcc>
__device__ __forceinline__ void store_tile_rows(const GemmArgs& p, const CUtensorMap& tmY, uint32_t t_row,
                                                uint8_t* ebuf, const float* colp, int n_tile0, int row0, float sa,
                                                int lane) {
    const float2 sa2 = make_float2(sa, sa);
    const uint64_t y_policy = make_l2_policy_evict_first();
#pragma unroll 1
    for (int c = 0; c < kBN / EPI_COLS; ++c) {
        const int n0 = n_tile0 + c * EPI_COLS;
        if (n0 >= p.N) break;  // uniform across the warp
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
}

template <int kAcc>
__global__ void __launch_bounds__(THREADS, 1)
    scaled_mm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmY, GemmArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + STAGES * A_STAGE_BYTES;
    uint8_t* sE = sB + STAGES * B_STAGE_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(sE + SMEM_EPI);
    uint64_t* empty = full + STAGES;
    uint64_t* tmem_full = empty + STAGES;
    uint64_t* tmem_empty = tmem_full + 2;
    uint64_t* drain = tmem_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int total_tiles = p.m_tiles * p.n_tiles;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tmem_full[i], 1);
            mbar_init(&tmem_empty[i], EPI_WARPS);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmY);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer
        if (lane == 0) {
            uint64_t pol_a, pol_b;
            l2_policies(p, pol_a, pol_b);
            int it = 0;
            int issued_phase[STAGES];
            for (int i = 0; i < STAGES; ++i) issued_phase[i] = -1;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                int tm, tn;
                tile_coords(t, p, tm, tn);
                for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                    const int st = it % STAGES;
                    const uint32_t ph = static_cast<uint32_t>(it / STAGES) & 1u;
                    if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag)) {
                        give_up(abort_flag, p.err, kErrGemmProducer);
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[st], A_STAGE_BYTES + B_STAGE_BYTES);
                    tma_load_2d_hint(sA + st * A_STAGE_BYTES, &tmA, kb * BK, tm * BM, &full[st], pol_a);
                    tma_load_2d_hint(sB + st * B_STAGE_BYTES, &tmB, kb * BK, tn * BN, &full[st], pol_b);
                    issued_phase[st] = static_cast<int>(ph);
                }
            }
            // Outstanding loads must land before the CTA may exit.
            for (int i = 0; i < STAGES; ++i)
                if (issued_phase[i] >= 0 && !mbar_wait(&full[i], static_cast<uint32_t>(issued_phase[i]), nullptr))
                    atomicOr(p.err, kErrGemmDrain);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int it = 0, tcount = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++tcount) {
                const int buf = tcount & 1;
                const uint32_t use = static_cast<uint32_t>(tcount >> 1);
                if (!mbar_wait(&tmem_empty[buf], (use & 1u) ^ 1u, abort_flag)) {
                    give_up(abort_flag, p.err, kErrGemmMma);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
                for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                    const int st = it % STAGES;
                    const uint32_t ph = static_cast<uint32_t>(it / STAGES) & 1u;
                    if (!mbar_wait(&full[st], ph, abort_flag)) {
                        give_up(abort_flag, p.err, kErrGemmMma);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t a_desc = sw128_kmajor_desc(sA + st * A_STAGE_BYTES);
                    const uint64_t b_desc = sw128_kmajor_desc(sB + st * B_STAGE_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        // advance the start address by k * 32 bytes inside the swizzle atom
                        const uint64_t koff = static_cast<uint64_t>((k * UMMA_K) >> 4);
                        mma_e4m3<kAcc == kAccS32>(d_tmem, a_desc + koff, b_desc + koff, make_idesc<kAcc>(BM, BN),
                                      (kb | k) != 0 ? 1u : 0u);
                    }
                    mma_commit(&empty[st]);
                }
                if (ok) mma_commit(&tmem_full[buf]);
            }
            // Every MMA issued above must finish before TMEM is freed.
            mma_commit(drain);
            if (!mbar_wait(drain, 0, nullptr)) atomicOr(p.err, kErrGemmDrain);
        }
    } else {
        // -------------------------------------------------------- epilogue
        const int ew = warp - 2;         // 0..3: staging buffers
        const int quarter = warp & 3;    // TMEM lanes this warp may read
        uint8_t* ebuf = sE + static_cast<size_t>(ew) * EPI_BUF_BYTES;
        float* colp = reinterpret_cast<float*>(sE + EPI_WARPS * EPI_BUF_BYTES + ew * COLP_BYTES);
        int tcount = 0;
        for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++tcount) {
            int tm, tn;
            tile_coords(t, p, tm, tn);
            stage_col_params<BN>(p, colp, tn * BN, lane);
            const int buf = tcount & 1;
            const uint32_t use = static_cast<uint32_t>(tcount >> 1);
            if (!mbar_wait_warp(&tmem_full[buf], use & 1u, abort_flag)) {
                if (lane == 0) give_up(abort_flag, p.err, kErrGemmEpilogue);
                break;
            }
            tc_fence_after();
            const int row0 = tm * BM + quarter * 32;
            const int m = row0 + lane;
            const float sa = (m < p.M) ? __ldg(p.s_a + m) : 0.0f;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(buf * BN);
            store_tile_rows<BN, kAcc>(p, tmY, t_row, ebuf, colp, tn * BN, row0, sa, lane);
            // All of this warp's TMEM reads of `buf` are complete: hand it back.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_empty[buf]);
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// MXFP8 block-scaled kernel (tcgen05.mma kind::mxf8f6f4.block_scale, one
// CTA per tile): the same roles as scaled_mm_kernel with 128 x 192 tiles.
// Each stage also brings the tile's E8M0 scale codes for its 4 K blocks --
// one 512-byte atom for the 128 rows of A, two for the 192 rows of B (the
// tile may start half-way into an atom) -- with plain bulk copies on the
// stage's "full" barrier.  The MMA thread copies them into TMEM with
// tcgen05.cp (32 x 128 bits, broadcast to the four lane quarters: TMEM
// column c of lane l holds the codes of row 32 c + l % 32 of the atom, one
// byte per K block), then issues the four K = 32 MMAs, each naming the byte
// of its K block (scale factor id).  tcgen05.cp and tcgen05.mma issued by one
// thread execute in order, so one TMEM copy of the scales serves every
// stage: the next stage's copy lands after the previous MMAs have read.
// TMEM: two 192-column accumulators (columns 0..383), A scales at 384..387,
// B scales at 388..395.  The epilogue applies only the bias (the scales are
// inside the accumulator).
constexpr int MX_BN = 192;
constexpr int MX_STAGES = 4;
constexpr int MX_B_STAGE_BYTES = MX_BN * BK;            // 24 KiB
constexpr int MX_SFA_BYTES = 512;                       // one atom: 128 rows x 4 K blocks
constexpr int MX_SFB_BYTES = 1024;                      // two atoms
constexpr uint32_t MX_SFA_COL = 2 * MX_BN;
constexpr uint32_t MX_SFB_COL = MX_SFA_COL + 4;
constexpr size_t MX_SMEM_RING =
    static_cast<size_t>(MX_STAGES) * (A_STAGE_BYTES + MX_B_STAGE_BYTES + MX_SFA_BYTES + MX_SFB_BYTES);
constexpr size_t MX_SMEM_BYTES = 1024 + MX_SMEM_RING + SMEM_EPI + SMEM_BARS;
static_assert(MX_SMEM_BYTES <= 232448, "shared memory budget exceeded");
static_assert(MX_SFB_COL + 8 <= 512, "TMEM budget exceeded");

// Instruction descriptor of the block-scaled MMA: E4M3 A and B (format 0),
// K-major, N >> 3 in bits 17-22, scale format E8M0 (bit 23), M >> 4 in bits
// 24-28; the scale factor ids of B (bits 4-5) and A (bits 29-30) are added
// per instruction.
constexpr uint32_t make_mx_idesc(int m, int n) {
    return (static_cast<uint32_t>(n >> 3) << 17) | (1u << 23) | (static_cast<uint32_t>(m >> 4) << 24);
}

struct MxArgs {
    const uint8_t* sf_a;  // scale-factor layout of A: atoms (kb, m / 128) at (kb * ra_a + m / 128) * 512
    const uint8_t* sf_w;
    int ra_a, ra_w;       // row atoms of A (ceil(M / 128)) and of W (ceil(N / 128))
};

__global__ void __launch_bounds__(THREADS, 1)
    mxfp8_mm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmY, GemmArgs p, MxArgs mx) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + MX_STAGES * A_STAGE_BYTES;
    uint8_t* sSFA = sB + MX_STAGES * MX_B_STAGE_BYTES;
    uint8_t* sSFB = sSFA + MX_STAGES * MX_SFA_BYTES;
    uint8_t* sE = sSFB + MX_STAGES * MX_SFB_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(sE + SMEM_EPI);
    uint64_t* empty = full + MX_STAGES;
    uint64_t* tmem_full = empty + MX_STAGES;
    uint64_t* tmem_empty = tmem_full + 2;
    uint64_t* drain = tmem_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int total_tiles = p.m_tiles * p.n_tiles;

    if (threadIdx.x == 0) {
        for (int i = 0; i < MX_STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tmem_full[i], 1);
            mbar_init(&tmem_empty[i], EPI_WARPS);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmY);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer
        if (lane == 0) {
            uint64_t pol_a, pol_b;
            l2_policies(p, pol_a, pol_b);
            int it = 0;
            int issued_phase[MX_STAGES];
            for (int i = 0; i < MX_STAGES; ++i) issued_phase[i] = -1;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                int tm, tn;
                tile_coords(t, p, tm, tn);
                const int a0 = (tn * MX_BN) >> 7;                    // first B row atom of the tile
                const uint32_t sfb_bytes = a0 + 1 < mx.ra_w ? 2 * 512 : 512;
                for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                    const int st = it % MX_STAGES;
                    const uint32_t ph = static_cast<uint32_t>(it / MX_STAGES) & 1u;
                    if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag)) {
                        give_up(abort_flag, p.err, kErrGemmProducer);
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[st], A_STAGE_BYTES + MX_B_STAGE_BYTES + MX_SFA_BYTES + sfb_bytes);
                    tma_load_2d_hint(sA + st * A_STAGE_BYTES, &tmA, kb * BK, tm * BM, &full[st], pol_a);
                    tma_load_2d_hint(sB + st * MX_B_STAGE_BYTES, &tmB, kb * BK, tn * MX_BN, &full[st], pol_b);
                    bulk_g2s(sSFA + st * MX_SFA_BYTES,
                             mx.sf_a + (static_cast<int64_t>(kb) * mx.ra_a + tm) * 512, MX_SFA_BYTES, &full[st]);
                    bulk_g2s(sSFB + st * MX_SFB_BYTES,
                             mx.sf_w + (static_cast<int64_t>(kb) * mx.ra_w + a0) * 512, sfb_bytes, &full[st]);
                    issued_phase[st] = static_cast<int>(ph);
                }
            }
            for (int i = 0; i < MX_STAGES; ++i)
                if (issued_phase[i] >= 0 && !mbar_wait(&full[i], static_cast<uint32_t>(issued_phase[i]), nullptr))
                    atomicOr(p.err, kErrGemmDrain);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t sfa_t = tmem_base + MX_SFA_COL;
            const uint32_t sfb_t = tmem_base + MX_SFB_COL;
            int it = 0, tcount = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++tcount) {
                int tm, tn;
                tile_coords(t, p, tm, tn);
                // B rows of the tile start 0 or 64 rows into their first atom:
                // skip that many 32-row TMEM columns of the B scales
                const uint32_t sfb_shift = static_cast<uint32_t>(((tn * MX_BN) & 127) >> 5);
                const int buf = tcount & 1;
                const uint32_t use = static_cast<uint32_t>(tcount >> 1);
                if (!mbar_wait(&tmem_empty[buf], (use & 1u) ^ 1u, abort_flag)) {
                    give_up(abort_flag, p.err, kErrGemmMma);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * MX_BN);
                for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                    const int st = it % MX_STAGES;
                    const uint32_t ph = static_cast<uint32_t>(it / MX_STAGES) & 1u;
                    if (!mbar_wait(&full[st], ph, abort_flag)) {
                        give_up(abort_flag, p.err, kErrGemmMma);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    tmem_cp_32x128b_warpx4(sfa_t, plain_rows16_desc(sSFA + st * MX_SFA_BYTES));
                    tmem_cp_32x128b_warpx4(sfb_t, plain_rows16_desc(sSFB + st * MX_SFB_BYTES));
                    tmem_cp_32x128b_warpx4(sfb_t + 4, plain_rows16_desc(sSFB + st * MX_SFB_BYTES + 512));
                    const uint64_t a_desc = sw128_kmajor_desc(sA + st * A_STAGE_BYTES);
                    const uint64_t b_desc = sw128_kmajor_desc(sB + st * MX_B_STAGE_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        const uint64_t koff = static_cast<uint64_t>((k * UMMA_K) >> 4);
                        const uint32_t id = static_cast<uint32_t>(k);
                        const uint32_t idesc = make_mx_idesc(BM, MX_BN) | (id << 29) | (id << 4);
                        mma_mxf8_block_scaled(d_tmem, a_desc + koff, b_desc + koff, idesc, sfa_t | (id << 30),
                                              (sfb_t + sfb_shift) | (id << 30), (kb | k) != 0 ? 1u : 0u);
                    }
                    mma_commit(&empty[st]);
                }
                if (ok) mma_commit(&tmem_full[buf]);
            }
            mma_commit(drain);
            if (!mbar_wait(drain, 0, nullptr)) atomicOr(p.err, kErrGemmDrain);
        }
    } else {
        // -------------------------------------------------------- epilogue
        const int ew = warp - 2;
        const int quarter = warp & 3;
        uint8_t* ebuf = sE + static_cast<size_t>(ew) * EPI_BUF_BYTES;
        float* colp = reinterpret_cast<float*>(sE + EPI_WARPS * EPI_BUF_BYTES + ew * COLP_BYTES);
        int tcount = 0;
        for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++tcount) {
            int tm, tn;
            tile_coords(t, p, tm, tn);
            stage_col_params<MX_BN, true>(p, colp, tn * MX_BN, lane);
            const int buf = tcount & 1;
            const uint32_t use = static_cast<uint32_t>(tcount >> 1);
            if (!mbar_wait_warp(&tmem_full[buf], use & 1u, abort_flag)) {
                if (lane == 0) give_up(abort_flag, p.err, kErrGemmEpilogue);
                break;
            }
            tc_fence_after();
            const int row0 = tm * BM + quarter * 32;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(buf * MX_BN);
            store_tile_rows<MX_BN, kAccF32>(p, tmY, t_row, ebuf, colp, tn * MX_BN, row0, 1.0f, lane);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_empty[buf]);
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

// ---------------------------------------------------------------------------
// CTA-pair kernel (cta_group::2): a cluster of two CTAs on two SMs computes a
// 256 x PBN tile.  CTA r of the pair loads rows [128 r, 128 r + 128) of the
// tile's A panel and rows [PBN/2 r, PBN/2 (r + 1)) of its B panel into its
// own shared memory; the even CTA's single MMA thread issues
// tcgen05.mma.cta_group::2 (M = 256, N = PBN, K = 32), which reads both
// CTAs' halves and leaves rows [128 r, 128 r + 128) of the accumulator in
// CTA r's TMEM.  Per CTA a stage is 16 KiB of A + PBN/2 x 128 B of B (32 KiB
// at PBN = 256 instead of 48 KiB), so six stages fit and each SM pulls a
// third less data from L2 per FLOP.  Both CTAs' loads complete on the even
// CTA's "full" barrier (which expects the bytes of both); the MMA thread
// releases each stage and each accumulator to both CTAs with a multicast
// commit; both CTAs' epilogue warps hand the accumulator back on the even
// CTA's "tmem_empty" barrier.  The epilogue is the same as above.
constexpr int PAIR_STAGES = 6;

template <int PBN>
struct PairCfg {
    static constexpr int kBHalf = PBN / 2;                      // B rows per CTA
    static constexpr int kAStage = 128 * BK;                    // 16 KiB
    static constexpr int kBStage = kBHalf * BK;
    static constexpr int kTmemCols = 512;                       // two PBN-column accumulators, power of 2
    static constexpr size_t kRing = static_cast<size_t>(PAIR_STAGES) * (kAStage + kBStage);
    static constexpr size_t kSmem = 1024 + kRing + SMEM_EPI + (2 * PAIR_STAGES + 4 + 1) * 8 + 16;
    static_assert(kSmem <= 232448, "shared memory budget exceeded");
    static_assert(2 * PBN <= kTmemCols, "two accumulators must fit in TMEM");
    static_assert(PBN % 64 == 0 && PBN >= 64 && PBN <= 256, "N tile");
};

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

template <int PBN, int kAcc>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    scaled_mm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                const __grid_constant__ CUtensorMap tmY, GemmArgs p) {
    using C = PairCfg<PBN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + PAIR_STAGES * C::kAStage;
    uint8_t* sE = sB + PAIR_STAGES * C::kBStage;
    uint64_t* full = reinterpret_cast<uint64_t*>(sE + SMEM_EPI);
    uint64_t* empty = full + PAIR_STAGES;
    uint64_t* tmem_full = empty + PAIR_STAGES;
    uint64_t* tmem_empty = tmem_full + 2;
    uint64_t* drain = tmem_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int cluster = blockIdx.x >> 1;
    const int n_clusters = gridDim.x >> 1;
    const int m_tiles = (p.M + 255) / 256;
    const int total_tiles = m_tiles * p.n_tiles;

    if (threadIdx.x == 0) {
        for (int i = 0; i < PAIR_STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tmem_full[i], 1);
            mbar_init(&tmem_empty[i], 2 * EPI_WARPS);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmY);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer
        if (lane == 0) {
            uint64_t pol_a, pol_b;
            l2_policies(p, pol_a, pol_b);
            int it = 0;
            int issued_phase[PAIR_STAGES];
            for (int i = 0; i < PAIR_STAGES; ++i) issued_phase[i] = -1;
            bool ok = true;
            int round = 0;
            for (int t = cluster; t < total_tiles && ok; t += n_clusters, ++round) {
                if (rank == 0) pace_round(p.round_ctr, round, total_tiles, n_clusters);
                int tm, tn;
                pair_tile_coords(t, m_tiles, p.n_tiles, p.group_m, p.band_n, tm, tn);
                const int a_row = tm * 256 + static_cast<int>(rank) * 128;
                const int b_row = tn * PBN + static_cast<int>(rank) * C::kBHalf;
                for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                    const int st = it % PAIR_STAGES;
                    const uint32_t ph = static_cast<uint32_t>(it / PAIR_STAGES) & 1u;
                    if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag)) {
                        give_up(abort_flag, p.err, kErrGemmProducer);
                        ok = false;
                        break;
                    }
                    const uint32_t full_leader = mapa_shared(smem_u32(&full[st]), 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full[st], 2 * (C::kAStage + C::kBStage));
                    tma_load_2d_pair(sA + st * C::kAStage, &tmA, kb * BK, a_row, full_leader, pol_a);
                    tma_load_2d_pair(sB + st * C::kBStage, &tmB, kb * BK, b_row, full_leader, pol_b);
                    issued_phase[st] = static_cast<int>(ph);
                }
                if (ok && rank == 0 && p.round_ctr != nullptr) atomicAdd(p.round_ctr, 1u);
            }
            // The even CTA's "full" barriers count both CTAs' loads: the even
            // producer waits for everything in flight before the final
            // cluster barrier lets either CTA exit.
            if (rank == 0) {
                for (int i = 0; i < PAIR_STAGES; ++i)
                    if (issued_phase[i] >= 0 &&
                        !mbar_wait(&full[i], static_cast<uint32_t>(issued_phase[i]), nullptr))
                        atomicOr(p.err, kErrGemmDrain);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------- MMA issuer (even CTA)
        if (lane == 0 && rank == 0) {
            int it = 0, tcount = 0;
            bool ok = true;
            for (int t = cluster; t < total_tiles && ok; t += n_clusters, ++tcount) {
                const int buf = tcount & 1;
                const uint32_t use = static_cast<uint32_t>(tcount >> 1);
                if (!mbar_wait(&tmem_empty[buf], (use & 1u) ^ 1u, abort_flag)) {
                    give_up(abort_flag, p.err, kErrGemmMma);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * PBN);
                for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                    const int st = it % PAIR_STAGES;
                    const uint32_t ph = static_cast<uint32_t>(it / PAIR_STAGES) & 1u;
                    if (!mbar_wait(&full[st], ph, abort_flag)) {
                        give_up(abort_flag, p.err, kErrGemmMma);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t a_desc = sw128_kmajor_desc(sA + st * C::kAStage);
                    const uint64_t b_desc = sw128_kmajor_desc(sB + st * C::kBStage);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        const uint64_t koff = static_cast<uint64_t>((k * UMMA_K) >> 4);
                        mma_e4m3_pair<kAcc == kAccS32>(d_tmem, a_desc + koff, b_desc + koff, make_idesc<kAcc>(256, PBN),
                                           (kb | k) != 0 ? 1u : 0u);
                    }
                    mma_commit_pair(&empty[st], 0x3);
                }
                if (ok) mma_commit_pair(&tmem_full[buf], 0x3);
            }
            mma_commit_pair(drain, 0x1);
            if (!mbar_wait(drain, 0, nullptr)) atomicOr(p.err, kErrGemmDrain);
        }
    } else {
        // ------------------------------------------- epilogue (both CTAs)
        const int ew = warp - 2;
        const int quarter = warp & 3;
        uint8_t* ebuf = sE + static_cast<size_t>(ew) * EPI_BUF_BYTES;
        float* colp = reinterpret_cast<float*>(sE + EPI_WARPS * EPI_BUF_BYTES + ew * COLP_BYTES);
        const uint32_t tmem_empty_leader0 = mapa_shared(smem_u32(&tmem_empty[0]), 0);
        const uint32_t tmem_empty_leader1 = mapa_shared(smem_u32(&tmem_empty[1]), 0);
        int tcount = 0;
        for (int t = cluster; t < total_tiles; t += n_clusters, ++tcount) {
            int tm, tn;
            pair_tile_coords(t, m_tiles, p.n_tiles, p.group_m, p.band_n, tm, tn);
            stage_col_params<PBN>(p, colp, tn * PBN, lane);
            const int buf = tcount & 1;
            const uint32_t use = static_cast<uint32_t>(tcount >> 1);
            if (!mbar_wait_warp(&tmem_full[buf], use & 1u, abort_flag)) {
                if (lane == 0) give_up(abort_flag, p.err, kErrGemmEpilogue);
                break;
            }
            tc_fence_after();
            const int row0 = tm * 256 + static_cast<int>(rank) * 128 + quarter * 32;
            const int m = row0 + lane;
            const float sa = (m < p.M) ? __ldg(p.s_a + m) : 0.0f;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(buf * PBN);
            store_tile_rows<PBN, kAcc>(p, tmY, t_row, ebuf, colp, tn * PBN, row0, sa, lane);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(buf == 0 ? tmem_empty_leader0 : tmem_empty_leader1);
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // neither CTA leaves while the pair may still touch its shared memory
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// MXFP8 CTA-pair kernel: a cluster of two CTAs computes a 256 x 192 tile with
// tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale (M = 256, N = 192).  As
// in scaled_mm_pair_kernel, CTA r loads rows [128 r, 128 r + 128) of the A
// panel and rows [96 r, 96 r + 96) of the B panel; in addition each CTA loads
// the scale atom of its own 128 A rows and both atoms that cover the tile's
// 192 B rows, all by TMA (the scale buffer viewed as rows of 512 bytes), all
// completing on the even CTA's "full" barrier.  The even CTA's MMA thread
// copies the scales of each stage into both CTAs' TMEM with one
// tcgen05.cp.cta_group::2 per atom (each CTA from its own shared memory), so
// the three copies per stage now serve twice the FLOPs of the one-CTA kernel.
constexpr int MXP_STAGES = 6;
constexpr int MXP_BHALF = MX_BN / 2;                     // 96 B rows per CTA
constexpr int MXP_B_STAGE_BYTES = MXP_BHALF * BK;        // 12 KiB
constexpr size_t MXP_SMEM_RING =
    static_cast<size_t>(MXP_STAGES) * (A_STAGE_BYTES + MXP_B_STAGE_BYTES + MX_SFA_BYTES + MX_SFB_BYTES);
constexpr size_t MXP_SMEM_BYTES = 1024 + MXP_SMEM_RING + SMEM_EPI + (2 * MXP_STAGES + 4 + 1) * 8 + 16;
static_assert(MXP_SMEM_BYTES <= 232448, "shared memory budget exceeded");

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    mxfp8_mm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmSA,
                         const __grid_constant__ CUtensorMap tmSB, GemmArgs p, MxArgs mx) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + MXP_STAGES * A_STAGE_BYTES;
    uint8_t* sSFA = sB + MXP_STAGES * MXP_B_STAGE_BYTES;
    uint8_t* sSFB = sSFA + MXP_STAGES * MX_SFA_BYTES;
    uint8_t* sE = sSFB + MXP_STAGES * MX_SFB_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(sE + SMEM_EPI);
    uint64_t* empty = full + MXP_STAGES;
    uint64_t* tmem_full = empty + MXP_STAGES;
    uint64_t* tmem_empty = tmem_full + 2;
    uint64_t* drain = tmem_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int cluster = blockIdx.x >> 1;
    const int n_clusters = gridDim.x >> 1;
    const int m_tiles = (p.M + 255) / 256;
    const int total_tiles = m_tiles * p.n_tiles;

    if (threadIdx.x == 0) {
        for (int i = 0; i < MXP_STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tmem_full[i], 1);
            mbar_init(&tmem_empty[i], 2 * EPI_WARPS);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmY);
        prefetch_tensormap(&tmSA);
        prefetch_tensormap(&tmSB);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer
        if (lane == 0) {
            uint64_t pol_a, pol_b;
            l2_policies(p, pol_a, pol_b);
            const uint64_t pol_sf = make_l2_policy_evict_last();
            int it = 0;
            int issued_phase[MXP_STAGES];
            for (int i = 0; i < MXP_STAGES; ++i) issued_phase[i] = -1;
            bool ok = true;
            int round = 0;
            for (int t = cluster; t < total_tiles && ok; t += n_clusters, ++round) {
                if (rank == 0) pace_round(p.round_ctr, round, total_tiles, n_clusters);
                int tm, tn;
                pair_tile_coords(t, m_tiles, p.n_tiles, p.group_m, p.band_n, tm, tn);
                const int a_row = tm * 256 + static_cast<int>(rank) * 128;
                const int b_row = tn * MX_BN + static_cast<int>(rank) * MXP_BHALF;
                const int a_atom = tm * 2 + static_cast<int>(rank);  // this CTA's 128-row scale panel
                const int b_atom = (tn * MX_BN) >> 7;                // first of the two B scale atoms
                for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                    const int st = it % MXP_STAGES;
                    const uint32_t ph = static_cast<uint32_t>(it / MXP_STAGES) & 1u;
                    if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag)) {
                        give_up(abort_flag, p.err, kErrGemmProducer);
                        ok = false;
                        break;
                    }
                    const uint32_t full_leader = mapa_shared(smem_u32(&full[st]), 0);
                    if (rank == 0)
                        mbar_arrive_expect_tx(&full[st],
                                              2 * (A_STAGE_BYTES + MXP_B_STAGE_BYTES + MX_SFA_BYTES + MX_SFB_BYTES));
                    tma_load_2d_pair(sA + st * A_STAGE_BYTES, &tmA, kb * BK, a_row, full_leader, pol_a);
                    tma_load_2d_pair(sB + st * MXP_B_STAGE_BYTES, &tmB, kb * BK, b_row, full_leader, pol_b);
                    // scale atoms: row kb * ra + atom of the [KA * RA, 128 words] view; rows past
                    // the end read as zeros (only rows or columns outside the problem use them)
                    tma_load_2d_pair(sSFA + st * MX_SFA_BYTES, &tmSA, 0, kb * mx.ra_a + a_atom, full_leader, pol_sf);
                    tma_load_2d_pair(sSFB + st * MX_SFB_BYTES, &tmSB, 0, kb * mx.ra_w + b_atom, full_leader, pol_sf);
                    issued_phase[st] = static_cast<int>(ph);
                }
                if (ok && rank == 0 && p.round_ctr != nullptr) atomicAdd(p.round_ctr, 1u);
            }
            if (rank == 0) {
                for (int i = 0; i < MXP_STAGES; ++i)
                    if (issued_phase[i] >= 0 &&
                        !mbar_wait(&full[i], static_cast<uint32_t>(issued_phase[i]), nullptr))
                        atomicOr(p.err, kErrGemmDrain);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------- MMA issuer (even CTA)
        if (lane == 0 && rank == 0) {
            const uint32_t sfa_t = tmem_base + MX_SFA_COL;
            const uint32_t sfb_t = tmem_base + MX_SFB_COL;
            int it = 0, tcount = 0;
            bool ok = true;
            for (int t = cluster; t < total_tiles && ok; t += n_clusters, ++tcount) {
                int tm, tn;
                pair_tile_coords(t, m_tiles, p.n_tiles, p.group_m, p.band_n, tm, tn);
                const uint32_t sfb_shift = static_cast<uint32_t>(((tn * MX_BN) & 127) >> 5);
                const int buf = tcount & 1;
                const uint32_t use = static_cast<uint32_t>(tcount >> 1);
                if (!mbar_wait(&tmem_empty[buf], (use & 1u) ^ 1u, abort_flag)) {
                    give_up(abort_flag, p.err, kErrGemmMma);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * MX_BN);
                for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                    const int st = it % MXP_STAGES;
                    const uint32_t ph = static_cast<uint32_t>(it / MXP_STAGES) & 1u;
                    if (!mbar_wait(&full[st], ph, abort_flag)) {
                        give_up(abort_flag, p.err, kErrGemmMma);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    tmem_cp_32x128b_warpx4_pair(sfa_t, plain_rows16_desc(sSFA + st * MX_SFA_BYTES));
                    tmem_cp_32x128b_warpx4_pair(sfb_t, plain_rows16_desc(sSFB + st * MX_SFB_BYTES));
                    tmem_cp_32x128b_warpx4_pair(sfb_t + 4, plain_rows16_desc(sSFB + st * MX_SFB_BYTES + 512));
                    const uint64_t a_desc = sw128_kmajor_desc(sA + st * A_STAGE_BYTES);
                    const uint64_t b_desc = sw128_kmajor_desc(sB + st * MXP_B_STAGE_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        const uint64_t koff = static_cast<uint64_t>((k * UMMA_K) >> 4);
                        const uint32_t id = static_cast<uint32_t>(k);
                        const uint32_t idesc = make_mx_idesc(256, MX_BN) | (id << 29) | (id << 4);
                        mma_mxf8_block_scaled_pair(d_tmem, a_desc + koff, b_desc + koff, idesc, sfa_t | (id << 30),
                                                   (sfb_t + sfb_shift) | (id << 30), (kb | k) != 0 ? 1u : 0u);
                    }
                    mma_commit_pair(&empty[st], 0x3);
                }
                if (ok) mma_commit_pair(&tmem_full[buf], 0x3);
            }
            mma_commit_pair(drain, 0x1);
            if (!mbar_wait(drain, 0, nullptr)) atomicOr(p.err, kErrGemmDrain);
        }
    } else {
        // ------------------------------------------- epilogue (both CTAs)
        const int ew = warp - 2;
        const int quarter = warp & 3;
        uint8_t* ebuf = sE + static_cast<size_t>(ew) * EPI_BUF_BYTES;
        float* colp = reinterpret_cast<float*>(sE + EPI_WARPS * EPI_BUF_BYTES + ew * COLP_BYTES);
        const uint32_t tmem_empty_leader0 = mapa_shared(smem_u32(&tmem_empty[0]), 0);
        const uint32_t tmem_empty_leader1 = mapa_shared(smem_u32(&tmem_empty[1]), 0);
        int tcount = 0;
        for (int t = cluster; t < total_tiles; t += n_clusters, ++tcount) {
            int tm, tn;
            pair_tile_coords(t, m_tiles, p.n_tiles, p.group_m, p.band_n, tm, tn);
            stage_col_params<MX_BN, true>(p, colp, tn * MX_BN, lane);
            const int buf = tcount & 1;
            const uint32_t use = static_cast<uint32_t>(tcount >> 1);
            if (!mbar_wait_warp(&tmem_full[buf], use & 1u, abort_flag)) {
                if (lane == 0) give_up(abort_flag, p.err, kErrGemmEpilogue);
                break;
            }
            tc_fence_after();
            const int row0 = tm * 256 + static_cast<int>(rank) * 128 + quarter * 32;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(buf * MX_BN);
            store_tile_rows<MX_BN, kAccF32>(p, tmY, t_row, ebuf, colp, tn * MX_BN, row0, 1.0f, lane);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(buf == 0 ? tmem_empty_leader0 : tmem_empty_leader1);
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 512);
    }
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

namespace {

// A wait that can only end by running out: the barrier expects one arrival
// that nothing makes.  Exercises the bounded wait the GEMM roles use (same
// helper, a shorter limit) and the error word that reports it.
__global__ void wait_selftest_kernel(uint64_t limit_ns, uint32_t* err) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort_flag, limit_ns)) atomicOr(err, kErrSelfTest);
}

template <int kAcc>
tfq_status launch_scaled_mm(const void* A, const float* s_a, const void* W, const float* s_w, const void* bias,
                            int64_t M, int64_t N, int64_t K, void* out, cudaStream_t stream, DeviceState* ds) {
    if (M == 0 || N == 0) return TFQ_OK;
    CUtensorMap tmA, tmY;
    tfq_status st = encode_tensor_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, K, M, K, BK, BM,
                                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != TFQ_OK) return st;
    st = encode_tensor_map_2d(&tmY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, out, N, M, N * 2, EPI_COLS, 32,
                              CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != TFQ_OK) return st;
    const int attr_idx = kAcc;
    if (!ds->gemm_attr_set[attr_idx]) {
        cudaError_t e = cudaFuncSetAttribute(scaled_mm_kernel<kAcc>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(SMEM_BYTES));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(scaled_mm_pair_kernel<256, kAcc>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(PairCfg<256>::kSmem));
        if (e != cudaSuccess) return fail(TFQ_ECUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        ds->gemm_attr_set[attr_idx] = true;
    }
    GemmArgs a;
    a.s_a = s_a;
    a.s_w = s_w;
    a.bias = static_cast<const uint16_t*>(bias);
    a.M = static_cast<int>(M);
    a.N = static_cast<int>(N);
    a.K = static_cast<int>(K);
    a.m_tiles = static_cast<int>((M + BM - 1) / BM);
    a.n_tiles = static_cast<int>((N + BN - 1) / BN);
    a.k_blocks = static_cast<int>((K + BK - 1) / BK);
    choose_raster(K, use_pair_kernel(M, ds->sm_count) ? 256 : BN, a.band_n, a.group_m);
    a.err = ds->err_word;
    a.round_ctr = nullptr;
    const int64_t tiles = static_cast<int64_t>(a.m_tiles) * a.n_tiles;
    if (tiles > INT32_MAX) return fail(TFQ_EUNSUPPORTED, "too many output tiles");
    if (use_pair_kernel(M, ds->sm_count)) {
        CUtensorMap tmBh;
        st = encode_tensor_map_2d(&tmBh, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, K, N, K, BK, PairCfg<256>::kBHalf,
                                  CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != TFQ_OK) return st;
        const int64_t pair_tiles = ((M + 255) / 256) * static_cast<int64_t>(a.n_tiles);
        const int clusters = static_cast<int>(std::min<int64_t>(pair_tiles, ds->sm_count / 2));
        a.round_ctr = take_round_counter(ds);
        if (a.round_ctr != nullptr) {
            const cudaError_t e = cudaMemsetAsync(a.round_ctr, 0, sizeof(unsigned), stream);
            if (e != cudaSuccess) return fail(TFQ_ECUDA, "clearing the round counter: %s", cudaGetErrorString(e));
        }
        scaled_mm_pair_kernel<256, kAcc><<<2 * clusters, THREADS, PairCfg<256>::kSmem, stream>>>(tmA, tmBh, tmY, a);
    } else {
        CUtensorMap tmB;
        st = encode_tensor_map_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, K, N, K, BK, BN,
                                  CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != TFQ_OK) return st;
        const int grid = static_cast<int>(std::min<int64_t>(tiles, ds->sm_count));
        scaled_mm_kernel<kAcc><<<grid, THREADS, SMEM_BYTES, stream>>>(tmA, tmB, tmY, a);
    }
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TFQ_OK : fail(TFQ_ECUDA, "GEMM launch: %s", cudaGetErrorString(e));
}

tfq_status launch_mxfp8_mm(const void* A, const uint8_t* sf_a, const void* W, const uint8_t* sf_w,
                           const void* bias, int64_t M, int64_t N, int64_t K, void* out, cudaStream_t stream,
                           DeviceState* ds) {
    if (M == 0 || N == 0) return TFQ_OK;
    CUtensorMap tmA, tmB, tmY;
    tfq_status st = encode_tensor_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, K, M, K, BK, BM,
                                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (st == TFQ_OK)
        st = encode_tensor_map_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, K, N, K, BK, MX_BN,
                                  CU_TENSOR_MAP_SWIZZLE_128B);
    if (st == TFQ_OK)
        st = encode_tensor_map_2d(&tmY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, out, N, M, N * 2, EPI_COLS, 32,
                                  CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != TFQ_OK) return st;
    if (!ds->gemm_attr_set[3]) {
        const cudaError_t e = cudaFuncSetAttribute(mxfp8_mm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   static_cast<int>(MX_SMEM_BYTES));
        if (e != cudaSuccess) return fail(TFQ_ECUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        ds->gemm_attr_set[3] = true;
    }
    GemmArgs a;
    a.s_a = nullptr;
    a.s_w = nullptr;
    a.bias = static_cast<const uint16_t*>(bias);
    a.M = static_cast<int>(M);
    a.N = static_cast<int>(N);
    a.K = static_cast<int>(K);
    a.m_tiles = static_cast<int>((M + BM - 1) / BM);
    a.n_tiles = static_cast<int>((N + MX_BN - 1) / MX_BN);
    a.k_blocks = static_cast<int>((K + BK - 1) / BK);
    choose_raster(K, MX_BN, a.band_n, a.group_m);
    a.err = ds->err_word;
    a.round_ctr = nullptr;
    MxArgs mx;
    mx.sf_a = sf_a;
    mx.sf_w = sf_w;
    mx.ra_a = static_cast<int>((M + 127) / 128);
    mx.ra_w = static_cast<int>((N + 127) / 128);
    const int64_t tiles = static_cast<int64_t>(a.m_tiles) * a.n_tiles;
    if (tiles > INT32_MAX) return fail(TFQ_EUNSUPPORTED, "too many output tiles");
    if (use_pair_kernel(M, ds->sm_count)) {
        // B halves of 96 rows; the scale buffers as [KA * RA, 128] 32-bit words
        // (one 512-byte atom per row): one atom for A, two for B per stage.
        CUtensorMap tmBh, tmSA, tmSB;
        const uint64_t ka = static_cast<uint64_t>((K + 127) / 128);
        st = encode_tensor_map_2d(&tmBh, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, K, N, K, BK, MXP_BHALF,
                                  CU_TENSOR_MAP_SWIZZLE_128B);
        if (st == TFQ_OK)
            st = encode_tensor_map_2d(&tmSA, CU_TENSOR_MAP_DATA_TYPE_UINT32, sf_a, 128, ka * mx.ra_a, 512, 128, 1,
                                      CU_TENSOR_MAP_SWIZZLE_NONE);
        if (st == TFQ_OK)
            st = encode_tensor_map_2d(&tmSB, CU_TENSOR_MAP_DATA_TYPE_UINT32, sf_w, 128, ka * mx.ra_w, 512, 128, 2,
                                      CU_TENSOR_MAP_SWIZZLE_NONE);
        if (st != TFQ_OK) return st;
        if (!ds->gemm_attr_set[4]) {
            const cudaError_t e = cudaFuncSetAttribute(mxfp8_mm_pair_kernel,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       static_cast<int>(MXP_SMEM_BYTES));
            if (e != cudaSuccess) return fail(TFQ_ECUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
            ds->gemm_attr_set[4] = true;
        }
        const int64_t pair_tiles = ((M + 255) / 256) * static_cast<int64_t>(a.n_tiles);
        const int clusters = static_cast<int>(std::min<int64_t>(pair_tiles, ds->sm_count / 2));
        a.round_ctr = take_round_counter(ds);
        if (a.round_ctr != nullptr) {
            const cudaError_t e = cudaMemsetAsync(a.round_ctr, 0, sizeof(unsigned), stream);
            if (e != cudaSuccess) return fail(TFQ_ECUDA, "clearing the round counter: %s", cudaGetErrorString(e));
        }
        mxfp8_mm_pair_kernel<<<2 * clusters, THREADS, MXP_SMEM_BYTES, stream>>>(tmA, tmBh, tmY, tmSA, tmSB, a, mx);
    } else {
        const int grid = static_cast<int>(std::min<int64_t>(tiles, ds->sm_count));
        mxfp8_mm_kernel<<<grid, THREADS, MX_SMEM_BYTES, stream>>>(tmA, tmB, tmY, a, mx);
    }
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TFQ_OK : fail(TFQ_ECUDA, "GEMM launch: %s", cudaGetErrorString(e));
}

}  // namespace

tfq_status launch_wait_selftest(uint64_t limit_ns, cudaStream_t stream, DeviceState* ds) {
    wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns, ds->err_word);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TFQ_OK : fail(TFQ_ECUDA, "self-test launch: %s", cudaGetErrorString(e));
}

tfq_status launch_scaled_fp8_gemm(const void* A, const float* s_a, const void* W, const float* s_w,
                                  const void* bias, int64_t M, int64_t N, int64_t K, void* out,
                                  cudaStream_t stream, DeviceState* ds) {
    return launch_scaled_mm<kAccF32>(A, s_a, W, s_w, bias, M, N, K, out, stream, ds);
}

tfq_status launch_scaled_fp8_gemm_f16acc(const void* A, const float* s_a, const void* W, const float* s_w,
                                         const void* bias, int64_t M, int64_t N, int64_t K, void* out,
                                         cudaStream_t stream, DeviceState* ds) {
    return launch_scaled_mm<kAccF16>(A, s_a, W, s_w, bias, M, N, K, out, stream, ds);
}

tfq_status launch_scaled_int8_gemm(const void* A, const float* s_a, const void* W, const float* s_w,
                                   const void* bias, int64_t M, int64_t N, int64_t K, void* out,
                                   cudaStream_t stream, DeviceState* ds) {
    return launch_scaled_mm<kAccS32>(A, s_a, W, s_w, bias, M, N, K, out, stream, ds);
}

tfq_status launch_mxfp8_gemm(const void* A, const uint8_t* sf_a, const void* W, const uint8_t* sf_w, const void* bias,
                             int64_t M, int64_t N, int64_t K, void* out, cudaStream_t stream, DeviceState* ds) {
    return launch_mxfp8_mm(A, sf_a, W, sf_w, bias, M, N, K, out, stream, ds);
}

}  // namespace tfq
