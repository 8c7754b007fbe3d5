// tfq_gemm_mx.cu -- MXFP8 block-scaled GEMM on 5th-generation tensor cores
// (tcgen05.mma kind::mxf8f6f4.block_scale, sm_100a).
//
// Computes out[m,n] = bf16_rn(sum_b 2^(sfa[m,b]-127) 2^(sfw[n,b]-127)
//                          sum_{k in block b} e4m3(A[m,k]) e4m3(W[n,k]) + bias[n])
// with one E8M0 scale per 32 consecutive K-elements of every row of A and of
// W: the MXFP8 format named on the TeleFuser "Quantization" page (section
// "Offline conversion": 32-value blocks, E8M0 scales).  The scale codes come
// in the layout the tensor cores read (512-byte atoms of 128 rows x 4 blocks,
// see include/tfq.h) and are applied by the MMA itself; the epilogue adds the
// bias.  Roles, barriers, raster and epilogue follow the scaled GEMM kernels.
#include "tfq_gemm_common.cuh"

namespace tfq {
namespace {

// Block-scaled MMA (MXFP8: E4M3 x E4M3, one E8M0 scale per 32 elements of K
// for every row of A and of B), single CTA.  sfa / sfb are TMEM addresses of
// the scale factors; their top two bits select the byte of each 32-bit TMEM
// cell (the scale of K block 0..3 of the stage), and must equal the scale
// factor ids carried in idesc.
__device__ __forceinline__ void mma_mxf8_block_scaled(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                      uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                                      uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// Copies 32 rows x 16 bytes of shared memory (row r at byte 16 r) into TMEM
// lanes 0..31, columns taddr..taddr+3, and the same data into lanes 32..63,
// 64..95 and 96..127 (the .warpx4 broadcast): the scale-factor staging of a
// block-scaled MMA.  Issued by the thread that issues the MMAs; it is
// ordered before them.
__device__ __forceinline__ void tmem_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// The same for a CTA pair (cta_group::2), issued by the even CTA: the MMA
// reads A and the A scales of each CTA from that CTA, and B from both; every
// CTA's TMEM holds the B scales of all N columns of the tile.
__device__ __forceinline__ void mma_mxf8_block_scaled_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                           uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// tmem_cp_32x128b_warpx4 for a CTA pair: in each CTA of the pair, from that
// CTA's shared memory at the descriptor's offset into its own TMEM.
__device__ __forceinline__ void tmem_cp_32x128b_warpx4_pair(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Shared-memory descriptor of an unswizzled K-major block of rows 16 bytes
// wide, stored contiguously: 8-row core matrices 128 bytes apart (stride
// byte offset), a single core-matrix column (leading byte offset unused).
__device__ __forceinline__ uint64_t plain_rows16_desc(const void* smem_rows) {
    const uint64_t addr = smem_u32(smem_rows);
    return ((addr >> 4) & 0x3FFFull) | ((128ull >> 4) << 32) | (1ull << 46);
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
    pdl_allow_next();
    pdl_wait();  // the set-up above may overlap the previous kernel; global memory only from here

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
// MXFP8 CTA-pair kernel: a cluster of two CTAs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale (M = 256, N = 256).  As
// in scaled_mm_pair_kernel, CTA r loads rows [128 r, 128 r + 128) of the A
// panel and rows [128 r, 128 r + 128) of the B panel; in addition each CTA
// loads the scale atom of its own 128 A rows and the two atoms of the tile's
// 256 B rows, all by TMA (the scale buffer viewed as rows of 512 bytes), all
// completing on the even CTA's "full" barrier.  The even CTA's MMA thread
// copies the scales of each stage into both CTAs' TMEM with one
// tcgen05.cp.cta_group::2 per atom (each CTA from its own shared memory).
//
// N = 256 with two accumulators and 12 scale columns needs 524 TMEM columns,
// 12 more than there are, so the two accumulators overlap by 32 columns:
// buffer 0 is columns [0, 256), buffer 1 [224, 480), the scales [480, 492).
// The epilogue of a tile reads the shared 32 columns first -- the last 64-
// column chunk of buffer 0, the first of buffer 1 -- and hands them back on
// an "overlap_free" barrier; the first MMA of the next tile (the other
// buffer) waits for that, besides the usual "tmem_empty" of its own buffer.
// Against 256 x 192 tiles with disjoint accumulators this gives each scale
// copy a third more FLOPs and each MMA its full width.
constexpr int MXP_BN = 256;
constexpr int MXP_OVERLAP = 32;                           // TMEM columns shared by the two accumulators
constexpr uint32_t MXP_BUF_STRIDE = MXP_BN - MXP_OVERLAP; // buffer b starts at column 224 b
constexpr uint32_t MXP_SFA_COL = MXP_BUF_STRIDE + MXP_BN; // 480
constexpr uint32_t MXP_SFB_COL = MXP_SFA_COL + 4;
static_assert(MXP_SFB_COL + 8 <= 512, "TMEM budget exceeded");
constexpr int MXP_STAGES = 6;
constexpr int MXP_BHALF = MXP_BN / 2;                    // 128 B rows per CTA
constexpr int MXP_B_STAGE_BYTES = MXP_BHALF * BK;        // 16 KiB
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
    __shared__ uint64_t overlap_free[2];  // epilogues of both CTAs: shared columns of buffer b read

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
        for (int i = 0; i < 2; ++i) mbar_init(&overlap_free[i], 2 * EPI_WARPS);
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
    pdl_allow_next();
    pdl_wait();  // the set-up above may overlap the previous kernel; global memory only from here

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
                const int b_row = tn * MXP_BN + static_cast<int>(rank) * MXP_BHALF;
                const int a_atom = tm * 2 + static_cast<int>(rank);  // this CTA's 128-row scale panel
                const int b_atom = tn * 2;                           // the tile's two B scale atoms
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
                pacing_done(p.round_ctr, n_clusters);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------- MMA issuer (even CTA)
        if (lane == 0 && rank == 0) {
            const uint32_t sfa_t = tmem_base + MXP_SFA_COL;
            const uint32_t sfb_t = tmem_base + MXP_SFB_COL;
            int it = 0, tcount = 0;
            bool ok = true;
            for (int t = cluster; t < total_tiles && ok; t += n_clusters, ++tcount) {
                const int buf = tcount & 1;
                const uint32_t use = static_cast<uint32_t>(tcount >> 1);
                // own buffer free (tile tcount - 2), and the columns it shares with the
                // other buffer read by the epilogue of tile tcount - 1
                if (!mbar_wait(&tmem_empty[buf], (use & 1u) ^ 1u, abort_flag) ||
                    (tcount >= 1 &&
                     !mbar_wait(&overlap_free[buf ^ 1], static_cast<uint32_t>((tcount - 1) >> 1) & 1u, abort_flag))) {
                    give_up(abort_flag, p.err, kErrGemmMma);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf) * MXP_BUF_STRIDE;
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
                        const uint32_t idesc = make_mx_idesc(256, MXP_BN) | (id << 29) | (id << 4);
                        mma_mxf8_block_scaled_pair(d_tmem, a_desc + koff, b_desc + koff, idesc, sfa_t | (id << 30),
                                                   sfb_t | (id << 30), (kb | k) != 0 ? 1u : 0u);
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
        const uint32_t overlap_leader0 = mapa_shared(smem_u32(&overlap_free[0]), 0);
        const uint32_t overlap_leader1 = mapa_shared(smem_u32(&overlap_free[1]), 0);
        const uint64_t y_policy = make_l2_policy_evict_first();
        constexpr int kChunks = MXP_BN / EPI_COLS;
        int tcount = 0;
        for (int t = cluster; t < total_tiles; t += n_clusters, ++tcount) {
            int tm, tn;
            pair_tile_coords(t, m_tiles, p.n_tiles, p.group_m, p.band_n, tm, tn);
            stage_col_params<MXP_BN, true>(p, colp, tn * MXP_BN, lane);
            const int buf = tcount & 1;
            const uint32_t use = static_cast<uint32_t>(tcount >> 1);
            if (!mbar_wait_warp(&tmem_full[buf], use & 1u, abort_flag)) {
                if (lane == 0) give_up(abort_flag, p.err, kErrGemmEpilogue);
                break;
            }
            tc_fence_after();
            const int row0 = tm * 256 + static_cast<int>(rank) * 128 + quarter * 32;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(buf) * MXP_BUF_STRIDE;
            // the chunk holding the shared columns first: last of buffer 0, first of buffer 1
            const int first = buf == 0 ? kChunks - 1 : 0;
            const float2 one2 = make_float2(1.0f, 1.0f);
            store_tile_chunk<MXP_BN, kAccF32>(p, tmY, t_row, ebuf, colp, tn * MXP_BN, row0, one2, y_policy, lane,
                                              first);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(buf == 0 ? overlap_leader0 : overlap_leader1);
#pragma unroll 1
            for (int c = 0; c < kChunks; ++c)
                if (c != first)
                    store_tile_chunk<MXP_BN, kAccF32>(p, tmY, t_row, ebuf, colp, tn * MXP_BN, row0, one2, y_policy,
                                                      lane, c);
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

}  // namespace

namespace {

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
        // 256-wide tiles; B halves of 128 rows; the scale buffers as [KA * RA, 128]
        // 32-bit words (one 512-byte atom per row): one atom for A, two for B per stage.
        a.n_tiles = static_cast<int>((N + MXP_BN - 1) / MXP_BN);
        choose_raster(K, MXP_BN, a.band_n, a.group_m);
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
        const cudaError_t el = launch_kernel(mxfp8_mm_pair_kernel, dim3(2 * clusters), dim3(THREADS), MXP_SMEM_BYTES,
                                             stream, tmA, tmBh, tmY, tmSA, tmSB, a, mx);
        if (el != cudaSuccess) return fail(TFQ_ECUDA, "GEMM launch: %s", cudaGetErrorString(el));
    } else {
        const int grid = static_cast<int>(std::min<int64_t>(tiles, ds->sm_count));
        const cudaError_t el = launch_kernel(mxfp8_mm_kernel, dim3(grid), dim3(THREADS), MX_SMEM_BYTES, stream, tmA,
                                             tmB, tmY, a, mx);
        if (el != cudaSuccess) return fail(TFQ_ECUDA, "GEMM launch: %s", cudaGetErrorString(el));
    }
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TFQ_OK : fail(TFQ_ECUDA, "GEMM launch: %s", cudaGetErrorString(e));
}

}  // namespace

tfq_status launch_mxfp8_gemm(const void* A, const uint8_t* sf_a, const void* W, const uint8_t* sf_w, const void* bias,
                             int64_t M, int64_t N, int64_t K, void* out, cudaStream_t stream, DeviceState* ds) {
    return launch_mxfp8_mm(A, sf_a, W, sf_w, bias, M, N, K, out, stream, ds);
}

}  // namespace tfq
