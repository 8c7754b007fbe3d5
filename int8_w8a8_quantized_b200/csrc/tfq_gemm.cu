// tfq_gemm.cu -- scaled FP8 GEMM with fused epilogue on 5th-generation
// tensor cores (tcgen05, sm_100a).
//
// Computes out[m,n] = bf16_rn(acc[m,n] * s_a[m] * s_w[n] + bias[n]) with
// acc[m,n] = sum_k e4m3(A[m,k]) * e4m3(W[n,k]) accumulated in fp32: the
// scaled GEMM of the TeleFuser "Quantization" page (sections "Scaled FP8
// checkpoints" and "tf-kernel FP8: online W8A8": per-token activation
// scales, per-output-channel weight scales, BF16 output).
//
// Two kernels: scaled_mm_pair_kernel (clusters of two CTAs computing 256 x
// 256 tiles with tcgen05.mma.cta_group::2; every problem of 512 rows or more)
// and scaled_mm_kernel (one CTA per 128 x 256 tile, smaller problems).  Both
// are templated on the operand kind: E4M3 with an fp32 or fp16 accumulator,
// or S8 with an s32 accumulator (the INT8 W8A8 path).
//
// One-CTA structure (one persistent CTA per SM, 192 threads; the pair kernel
// below follows it):
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
// Tiles are visited in bands of N tiles holding ~40 MB of weight, each band
// sweeping every M tile, so that the CTAs running at the same time share the
// band's weight panels (kept in L2) and each activation panel; the pair
// kernel also keeps its clusters within one tile of each other (pacing,
// see tfq_gemm_common.cuh) and runs a last round of at most half as many
// tiles as clusters as half-width (256 x 128) tiles.  M and N tails are handled by
// TMA (zero fill on load, clipping on store); K tails by zero fill.
// Every wait is bounded (see tfq_ptx.cuh); a CTA that gives up records it in
// the error word, drains its own outstanding copies and MMAs, frees TMEM and
// returns.
#include "tfq_gemm_common.cuh"
#include "tfq_quant_row.cuh"

namespace tfq {
namespace {

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
    pdl_allow_next();
    pdl_wait();  // the set-up above may overlap the previous kernel; global memory only from here

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

// The CTA-pair kernel that quantizes its own activations (kQuant != 0) adds
// QUANT_WARPS quantizer warps to every CTA.  They take rows of the bf16
// activations in increasing order from a counter shared by the whole grid,
// quantize each (one warp per row: max |x|, the fp32 scale, the E4M3 codes,
// exactly as the row quantizer kernels do) into the A operand and the row
// scales, and publish each finished row on its 128-row share's counter.
// They wait for nothing, so they always finish; the producers and the
// epilogues wait (bounded) for the shares they need.  The tensor cores of an
// SM run the MMAs of the current tiles while its quantizer warps, with
// those of every other SM, stream the rows of the coming tiles.
// Measured on B200 this overlap does not pay: the GEMM slows down by about
// the quantizer's own time (the quantizer's loads and stores share the SM's
// memory path with the operand traffic of the MMAs, and under the power cap
// the same work costs the same energy), so the row quantizer followed by the
// plain GEMM stays the default path; this variant is kept, parity-tested,
// as the measured alternative.
// kQuant: 0 = operands given quantized; 1 = E4M3 rows, qmax an E4M3 value
// (no clamp needed); 2 = E4M3 rows with the clamp to +-qmax.
#ifndef TFQ_QUANT_WARPS
#define TFQ_QUANT_WARPS 8  // measured on B200: 8 beat 4 (the warps are latency bound, one row at a time)
#endif
constexpr int QUANT_WARPS = TFQ_QUANT_WARPS;
constexpr int QUANT_SEG = 20;  // 16-byte units per lane per segment: a K = 5120 row in one pass

template <int kQuant>
constexpr int pair_threads() {
    return THREADS + (kQuant != 0 ? QUANT_WARPS * 32 : 0);
}

// Rows of the 128-row share of A starting at row0 that must be quantized
// before they may be read (0 past the end of M).
__device__ __forceinline__ unsigned share_rows(const GemmArgs& p, int row0) {
    return row0 >= p.M ? 0u : static_cast<unsigned>(min(128, p.M - row0));
}

// Waits (bounded; one thread) until the share of A starting at row0 is
// quantized: an acquire load of its counter, so that this thread's later
// reads see the codes and scales written by the quantizer warps, then a
// proxy fence, so that its later TMA loads (the async proxy) see them too.
__device__ __forceinline__ bool wait_share_quantized(const GemmArgs& p, int row0, volatile int* abort) {
    const unsigned need = share_rows(p, row0);
    if (need == 0) return true;
    const unsigned* ctr = p.q_share_rows + row0 / 128;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 0; i < TFQ_WAIT_LIMIT_POLLS; ++i) {
        unsigned v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
        if (v >= need) {
            asm volatile("fence.proxy.async.global;" ::: "memory");
            return true;
        }
        if ((i & 15u) == 15u) {
            if (abort != nullptr && *abort != 0) return false;
            if (globaltimer_ns() - t0 > TFQ_WAIT_LIMIT_NS) return false;
        }
        __nanosleep(256);
    }
    return false;
}

// The quantizer warps' loop (see above).
template <int kQuant>
__device__ __forceinline__ void quantize_rows_for_gemm(const GemmArgs& p, int lane) {
    const int units = p.K >> 3;
    const uint64_t keep = l2_policy_evict_last(), drop = l2_policy_evict_first();
    for (;;) {
        unsigned r = 0;
        if (lane == 0) r = atomicAdd(p.q_next_row, 1u);
        r = __shfl_sync(0xFFFFFFFFu, r, 0);
        if (r >= static_cast<unsigned>(p.M)) break;
        const size_t off = static_cast<size_t>(r) * static_cast<size_t>(units);
        quantize_row_warp<false, kQuant == 2, QUANT_SEG>(p.qx + off, units, p.qmax,
                                                        reinterpret_cast<uint2*>(p.qa + off * 8), p.qs + r, lane,
                                                        keep, drop);
        // Publish the row: each lane's stores are made visible to the async
        // proxy (the readers' TMA loads), the warp barrier orders them before
        // lane 0's release increment of the share counter (a release is
        // cumulative over the writes it has observed).  A full fence per
        // lane instead measured 10 % slower on the image-DiT Q projection.
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __syncwarp();
        if (lane == 0)
            asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(p.q_share_rows + r / 128) : "memory");
    }
}

// Tensor maps of the CTA-pair kernel per Linear (see GemmArgs::n_lin): the
// weight with 128-row boxes (b) and 64-row boxes (bq, the half-width tiles of
// a split last round), and the output (y).
struct PairMaps {
    CUtensorMap b[kMaxLinears];
    CUtensorMap bq[kMaxLinears];
    CUtensorMap y[kMaxLinears];
};

// One Linear's operands on the host side: weight codes [N, K], column scales,
// bias (may be null), N, output [M, N].
struct LinearOperands {
    const void* W;
    const float* s_w;
    const void* bias;
    int64_t N;
    void* out;
};

template <int PBN, int kAcc, int kQuant = 0>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair_threads<kQuant>(), 1)
    scaled_mm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ PairMaps maps,
                          GemmArgs p) {
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
        for (int i = 0; i < p.n_lin; ++i) {
            prefetch_tensormap(&maps.b[i]);
            if (p.tail_halves) prefetch_tensormap(&maps.bq[i]);
            prefetch_tensormap(&maps.y[i]);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_allow_next();
    pdl_wait();  // the set-up above may overlap the previous kernel; global memory only from here

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer
        if (lane == 0) {
            uint64_t pol_a, pol_b;
            l2_policies(p, pol_a, pol_b);
            int it = 0;
            int issued_phase[PAIR_STAGES];
            for (int i = 0; i < PAIR_STAGES; ++i) issued_phase[i] = -1;
            bool ok = true;
            int round = 0, t, half;
            for (int w = cluster; ok && pair_work_item(w, total_tiles, n_clusters, p.tail_halves, t, half);
                 w += n_clusters, ++round) {
                if (rank == 0) pace_round(p.round_ctr, round, total_tiles, n_clusters);
                int tm, tn_all, lin, tn;
                pair_tile_coords(t, m_tiles, p.n_tiles, p.group_m, p.band_n, tm, tn_all);
                split_linear_tile(p, tn_all, lin, tn);
                // a half tile: PBN / 2 columns, PBN / 4 B rows per CTA (bq's box)
                const int b_rows = half < 0 ? C::kBHalf : C::kBHalf / 2;
                const CUtensorMap* tmb = half < 0 ? &maps.b[lin] : &maps.bq[lin];
                const uint32_t stage_tx = 2 * static_cast<uint32_t>(C::kAStage + b_rows * BK);
                const int a_row = tm * 256 + static_cast<int>(rank) * 128;
                const int b_row = tn * PBN + (half > 0 ? PBN / 2 : 0) + static_cast<int>(rank) * b_rows;
                if constexpr (kQuant != 0) {
                    if (!wait_share_quantized(p, a_row, abort_flag)) {
                        give_up(abort_flag, p.err, kErrGemmProducer);
                        ok = false;
                        break;
                    }
                }
                for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                    const int st = it % PAIR_STAGES;
                    const uint32_t ph = static_cast<uint32_t>(it / PAIR_STAGES) & 1u;
                    if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag)) {
                        give_up(abort_flag, p.err, kErrGemmProducer);
                        ok = false;
                        break;
                    }
                    const uint32_t full_leader = mapa_shared(smem_u32(&full[st]), 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full[st], stage_tx);
                    tma_load_2d_pair(sA + st * C::kAStage, &tmA, kb * BK, a_row, full_leader, pol_a);
                    tma_load_2d_pair(sB + st * C::kBStage, tmb, kb * BK, b_row, full_leader, pol_b);
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
                pacing_done(p.round_ctr, n_clusters);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------- MMA issuer (even CTA)
        if (lane == 0 && rank == 0) {
            int it = 0, tcount = 0, t, half;
            bool ok = true;
            for (int w = cluster; ok && pair_work_item(w, total_tiles, n_clusters, p.tail_halves, t, half);
                 w += n_clusters, ++tcount) {
                const int buf = tcount & 1;
                const uint32_t use = static_cast<uint32_t>(tcount >> 1);
                if (!mbar_wait(&tmem_empty[buf], (use & 1u) ^ 1u, abort_flag)) {
                    give_up(abort_flag, p.err, kErrGemmMma);
                    break;
                }
                tc_fence_after();
                const uint32_t idesc = make_idesc<kAcc>(256, half < 0 ? PBN : PBN / 2);
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
                        mma_e4m3_pair<kAcc == kAccS32>(d_tmem, a_desc + koff, b_desc + koff, idesc,
                                                       (kb | k) != 0 ? 1u : 0u);
                    }
                    mma_commit_pair(&empty[st], 0x3);
                }
                if (ok) mma_commit_pair(&tmem_full[buf], 0x3);
            }
            mma_commit_pair(drain, 0x1);
            if (!mbar_wait(drain, 0, nullptr)) atomicOr(p.err, kErrGemmDrain);
        }
    } else if (warp < 2 + EPI_WARPS) {
        // ------------------------------------------- epilogue (both CTAs)
        const int ew = warp - 2;
        const int quarter = warp & 3;
        uint8_t* ebuf = sE + static_cast<size_t>(ew) * EPI_BUF_BYTES;
        float* colp = reinterpret_cast<float*>(sE + EPI_WARPS * EPI_BUF_BYTES + ew * COLP_BYTES);
        const uint32_t tmem_empty_leader0 = mapa_shared(smem_u32(&tmem_empty[0]), 0);
        const uint32_t tmem_empty_leader1 = mapa_shared(smem_u32(&tmem_empty[1]), 0);
        int tcount = 0, t, half;
        for (int w = cluster; pair_work_item(w, total_tiles, n_clusters, p.tail_halves, t, half);
             w += n_clusters, ++tcount) {
            int tm, tn_all, lin, tn;
            pair_tile_coords(t, m_tiles, p.n_tiles, p.group_m, p.band_n, tm, tn_all);
            split_linear_tile(p, tn_all, lin, tn);
            const GemmArgs pl = linear_args(p, lin);
            const int n0 = tn * PBN + (half > 0 ? PBN / 2 : 0);
            stage_col_params<PBN>(pl, colp, n0, lane);
            const int row0 = tm * 256 + static_cast<int>(rank) * 128 + quarter * 32;
            const int m = row0 + lane;
            float sa;
            if constexpr (kQuant != 0) {
                // the row scales come from this launch's quantizer warps: wait
                // for the share (it is complete before the tile's MMAs run)
                int ok = 1;
                if (lane == 0) ok = wait_share_quantized(p, row0 - quarter * 32, abort_flag) ? 1 : 0;
                if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) {
                    if (lane == 0) give_up(abort_flag, p.err, kErrGemmEpilogue);
                    break;
                }
                __syncwarp();
                sa = 0.0f;
                if (m < p.M) asm volatile("ld.relaxed.gpu.global.f32 %0, [%1];" : "=f"(sa) : "l"(p.qs + m) : "memory");
            } else {
                sa = (m < p.M) ? __ldg(p.s_a + m) : 0.0f;
            }
            const int buf = tcount & 1;
            const uint32_t use = static_cast<uint32_t>(tcount >> 1);
            if (!mbar_wait_warp(&tmem_full[buf], use & 1u, abort_flag)) {
                if (lane == 0) give_up(abort_flag, p.err, kErrGemmEpilogue);
                break;
            }
            tc_fence_after();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(buf * PBN);
            store_tile_rows<PBN, kAcc>(pl, maps.y[lin], t_row, ebuf, colp, n0, row0, sa, lane,
                                       half < 0 ? PBN : PBN / 2);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(buf == 0 ? tmem_empty_leader0 : tmem_empty_leader1);
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    } else {
        // ------------------------------------ quantizer warps (kQuant only)
        if constexpr (kQuant != 0) quantize_rows_for_gemm<kQuant>(p, lane);
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

// Opt-in shared memory of the scaled GEMM kernels of one accumulator kind (once per device).
template <int kAcc>
tfq_status set_gemm_attributes(DeviceState* ds) {
    if (ds->gemm_attr_set[kAcc]) return TFQ_OK;
    cudaError_t e = cudaFuncSetAttribute(scaled_mm_kernel<kAcc>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(SMEM_BYTES));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(scaled_mm_pair_kernel<256, kAcc>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(PairCfg<256>::kSmem));
    if (e != cudaSuccess) return fail(TFQ_ECUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    ds->gemm_attr_set[kAcc] = true;
    return TFQ_OK;
}

// The tensor maps and the Linear table of the CTA-pair kernel for n Linears
// that share A (their N tiles concatenated in order).
tfq_status pair_linear_setup(const LinearOperands* lins, int n, int64_t M, int64_t K, PairMaps& maps,
                             GemmArgs& a) {
    constexpr int kPBN = 256;
    using C = PairCfg<kPBN>;
    int tiles = 0;
    for (int i = 0; i < n; ++i) {
        const LinearOperands& l = lins[i];
        tfq_status st = encode_tensor_map_2d(&maps.b[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, l.W, K, l.N, K, BK,
                                             C::kBHalf, CU_TENSOR_MAP_SWIZZLE_128B);
        if (st == TFQ_OK)
            st = encode_tensor_map_2d(&maps.bq[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, l.W, K, l.N, K, BK, C::kBHalf / 2,
                                      CU_TENSOR_MAP_SWIZZLE_128B);
        if (st == TFQ_OK)
            st = encode_tensor_map_2d(&maps.y[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, l.out, l.N, M, l.N * 2, EPI_COLS,
                                      32, CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != TFQ_OK) return st;
        a.lin_tile0[i] = tiles;
        a.lin_s_w[i] = l.s_w;
        a.lin_bias[i] = static_cast<const uint16_t*>(l.bias);
        a.lin_N[i] = static_cast<int>(l.N);
        tiles += static_cast<int>((l.N + kPBN - 1) / kPBN);
    }
    for (int i = n; i <= kMaxLinears; ++i) a.lin_tile0[i] = tiles;
    a.n_lin = n;
    a.n_tiles = tiles;
    a.s_w = lins[0].s_w;
    a.bias = static_cast<const uint16_t*>(lins[0].bias);
    a.N = static_cast<int>(lins[0].N);
    return TFQ_OK;
}

// n Linears that share A (n = 1: the plain GEMM) as one launch of the
// CTA-pair kernel (M >= TFQ_GEMM_PAIR_MIN_M).
template <int kAcc>
tfq_status launch_pair_linears(const void* A, const float* s_a, int64_t M, int64_t K, const LinearOperands* lins,
                               int n, cudaStream_t stream, DeviceState* ds) {
    tfq_status st = set_gemm_attributes<kAcc>(ds);
    if (st != TFQ_OK) return st;
    CUtensorMap tmA;
    st = encode_tensor_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, K, M, K, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != TFQ_OK) return st;
    PairMaps maps = {};
    GemmArgs a;
    st = pair_linear_setup(lins, n, M, K, maps, a);
    if (st != TFQ_OK) return st;
    a.s_a = s_a;
    a.M = static_cast<int>(M);
    a.K = static_cast<int>(K);
    a.m_tiles = static_cast<int>((M + BM - 1) / BM);
    a.k_blocks = static_cast<int>((K + BK - 1) / BK);
    choose_raster(K, 256, a.band_n, a.group_m);
    a.err = ds->err_word;
    const int64_t pair_tiles = ((M + 255) / 256) * static_cast<int64_t>(a.n_tiles);
    if (pair_tiles > INT32_MAX) return fail(TFQ_EUNSUPPORTED, "too many output tiles");
    const int clusters = static_cast<int>(std::min<int64_t>(pair_tiles, ds->sm_count / 2));
    a.tail_halves = choose_tail_halves(pair_tiles, clusters);
    a.round_ctr = take_round_counter(ds);
    const cudaError_t el = launch_kernel(scaled_mm_pair_kernel<256, kAcc>, dim3(2 * clusters), dim3(THREADS),
                                         PairCfg<256>::kSmem, stream, tmA, maps, a);
    if (el != cudaSuccess) return fail(TFQ_ECUDA, "GEMM launch: %s", cudaGetErrorString(el));
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TFQ_OK : fail(TFQ_ECUDA, "GEMM launch: %s", cudaGetErrorString(e));
}

template <int kAcc>
tfq_status launch_scaled_mm(const void* A, const float* s_a, const void* W, const float* s_w, const void* bias,
                            int64_t M, int64_t N, int64_t K, void* out, cudaStream_t stream, DeviceState* ds) {
    if (M == 0 || N == 0) return TFQ_OK;
    if (use_pair_kernel(M, ds->sm_count)) {
        const LinearOperands lin = {W, s_w, bias, N, out};
        return launch_pair_linears<kAcc>(A, s_a, M, K, &lin, 1, stream, ds);
    }
    CUtensorMap tmA, tmY;
    tfq_status st = encode_tensor_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, K, M, K, BK, BM,
                                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != TFQ_OK) return st;
    st = encode_tensor_map_2d(&tmY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, out, N, M, N * 2, EPI_COLS, 32,
                              CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != TFQ_OK) return st;
    st = set_gemm_attributes<kAcc>(ds);
    if (st != TFQ_OK) return st;
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
    choose_raster(K, BN, a.band_n, a.group_m);
    a.err = ds->err_word;
    a.round_ctr = nullptr;
    const int64_t tiles = static_cast<int64_t>(a.m_tiles) * a.n_tiles;
    if (tiles > INT32_MAX) return fail(TFQ_EUNSUPPORTED, "too many output tiles");
    CUtensorMap tmB;
    st = encode_tensor_map_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, K, N, K, BK, BN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != TFQ_OK) return st;
    const int grid = static_cast<int>(std::min<int64_t>(tiles, ds->sm_count));
    const cudaError_t el = launch_kernel(scaled_mm_kernel<kAcc>, dim3(grid), dim3(THREADS), SMEM_BYTES, stream, tmA,
                                         tmB, tmY, a);
    if (el != cudaSuccess) return fail(TFQ_ECUDA, "GEMM launch: %s", cudaGetErrorString(el));
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TFQ_OK : fail(TFQ_ECUDA, "GEMM launch: %s", cudaGetErrorString(e));
}

}  // namespace

tfq_status launch_wait_selftest(uint64_t limit_ns, cudaStream_t stream, DeviceState* ds) {
    wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns, ds->err_word);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TFQ_OK : fail(TFQ_ECUDA, "self-test launch: %s", cudaGetErrorString(e));
}

size_t quant_gemm_workspace_bytes(int64_t M) {
    const size_t words = 32 + static_cast<size_t>((M + 127) / 128);
    return (words * sizeof(unsigned) + 255) / 256 * 256;
}

tfq_status launch_quant_scaled_fp8_gemm(const void* x, int64_t M, int64_t K, float qmax, bool clamp, const void* W,
                                        const float* s_w, const void* bias, int64_t N, void* A, float* s_a,
                                        void* out, void* workspace, cudaStream_t stream, DeviceState* ds) {
    if (M == 0) return TFQ_OK;
    if (!use_pair_kernel(M, ds->sm_count) || N == 0) {
        // Below the CTA-pair size: the row quantizer, then the GEMM.
        tfq_status st = launch_quant_rows(x, M, K, qmax, false, A, s_a, stream, ds);
        if (st != TFQ_OK || N == 0) return st;
        return launch_scaled_mm<kAccF32>(A, s_a, W, s_w, bias, M, N, K, out, stream, ds);
    }
    constexpr int kPBN = 256;
    using C = PairCfg<kPBN>;
    // The row counter (word 0) and the per-share counters (from word 32)
    // start at zero.
    cudaError_t e = cudaMemsetAsync(workspace, 0, quant_gemm_workspace_bytes(M), stream);
    if (e != cudaSuccess) return fail(TFQ_ECUDA, "clearing the workspace: %s", cudaGetErrorString(e));
    CUtensorMap tmA;
    tfq_status st = encode_tensor_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, K, M, K, BK, BM,
                                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != TFQ_OK) return st;
    PairMaps maps = {};
    GemmArgs a;
    const LinearOperands lin = {W, s_w, bias, N, out};
    st = pair_linear_setup(&lin, 1, M, K, maps, a);
    if (st != TFQ_OK) return st;
    auto kernel = clamp ? scaled_mm_pair_kernel<kPBN, kAccF32, 2> : scaled_mm_pair_kernel<kPBN, kAccF32, 1>;
    if (!ds->gemm_attr_set[5]) {
        e = cudaFuncSetAttribute(scaled_mm_pair_kernel<kPBN, kAccF32, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(C::kSmem));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(scaled_mm_pair_kernel<kPBN, kAccF32, 2>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::kSmem));
        if (e != cudaSuccess) return fail(TFQ_ECUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        ds->gemm_attr_set[5] = true;
    }
    a.s_a = s_a;
    a.M = static_cast<int>(M);
    a.K = static_cast<int>(K);
    a.m_tiles = static_cast<int>((M + BM - 1) / BM);
    a.k_blocks = static_cast<int>((K + BK - 1) / BK);
    choose_raster(K, kPBN, a.band_n, a.group_m);
    a.err = ds->err_word;
    const int64_t pair_tiles = ((M + 255) / 256) * static_cast<int64_t>(a.n_tiles);
    if (pair_tiles > INT32_MAX) return fail(TFQ_EUNSUPPORTED, "too many output tiles");
    const int clusters = static_cast<int>(std::min<int64_t>(pair_tiles, ds->sm_count / 2));
    a.tail_halves = choose_tail_halves(pair_tiles, clusters);
    a.round_ctr = take_round_counter(ds);
    unsigned* ws = static_cast<unsigned*>(workspace);
    a.qx = static_cast<const uint4*>(x);
    a.qa = static_cast<uint8_t*>(A);
    a.qs = s_a;
    a.q_next_row = ws;
    a.q_share_rows = ws + 32;
    a.qmax = qmax;
    e = launch_kernel(kernel, dim3(2 * clusters), dim3(pair_threads<1>()), C::kSmem, stream, tmA, maps, a);
    if (e != cudaSuccess) return fail(TFQ_ECUDA, "GEMM launch: %s", cudaGetErrorString(e));
    e = cudaGetLastError();
    return e == cudaSuccess ? TFQ_OK : fail(TFQ_ECUDA, "GEMM launch: %s", cudaGetErrorString(e));
}

tfq_status launch_scaled_fp8_gemm(const void* A, const float* s_a, const void* W, const float* s_w,
                                  const void* bias, int64_t M, int64_t N, int64_t K, void* out,
                                  cudaStream_t stream, DeviceState* ds) {
    return launch_scaled_mm<kAccF32>(A, s_a, W, s_w, bias, M, N, K, out, stream, ds);
}

namespace {

template <int kAcc>
tfq_status launch_gemm_multi(const void* A, const float* s_a, int64_t M, int64_t K, int n, const void* const* W,
                             const float* const* s_w, const void* const* bias, const int64_t* N, void* const* out,
                             cudaStream_t stream, DeviceState* ds) {
    if (M == 0) return TFQ_OK;
    LinearOperands lins[kMaxLinears];
    int m = 0;
    for (int i = 0; i < n; ++i)
        if (N[i] > 0) lins[m++] = {W[i], s_w[i], bias != nullptr ? bias[i] : nullptr, N[i], out[i]};
    if (m == 0) return TFQ_OK;
    if (!use_pair_kernel(M, ds->sm_count)) {  // one-CTA kernel, one launch per Linear
        for (int i = 0; i < m; ++i) {
            const tfq_status st = launch_scaled_mm<kAcc>(A, s_a, lins[i].W, lins[i].s_w, lins[i].bias, M, lins[i].N,
                                                         K, lins[i].out, stream, ds);
            if (st != TFQ_OK) return st;
        }
        return TFQ_OK;
    }
    return launch_pair_linears<kAcc>(A, s_a, M, K, lins, m, stream, ds);
}

}  // namespace

tfq_status launch_scaled_fp8_gemm_multi(const void* A, const float* s_a, int64_t M, int64_t K, int n,
                                        const void* const* W, const float* const* s_w, const void* const* bias,
                                        const int64_t* N, void* const* out, cudaStream_t stream, DeviceState* ds) {
    return launch_gemm_multi<kAccF32>(A, s_a, M, K, n, W, s_w, bias, N, out, stream, ds);
}

tfq_status launch_scaled_int8_gemm_multi(const void* A, const float* s_a, int64_t M, int64_t K, int n,
                                         const void* const* W, const float* const* s_w, const void* const* bias,
                                         const int64_t* N, void* const* out, cudaStream_t stream, DeviceState* ds) {
    return launch_gemm_multi<kAccS32>(A, s_a, M, K, n, W, s_w, bias, N, out, stream, ds);
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

}  // namespace tfq
