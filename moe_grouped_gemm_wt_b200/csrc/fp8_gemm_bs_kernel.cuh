// fp8_gemm_bs_kernel.cuh -- the UE8M0 block-scaled mode of the FP8 GEMM on
// sm_100a (dense, contiguous-grouped and masked-grouped layouts).
//
// Method: the SM100 path of the DeepGEMM pages takes its scaling factors as
// packed UE8M0, four to an int (hada.io summary, section "Giao dien GEMM va
// rang buoc layout").  With power-of-two scales the tensor core applies them
// itself: tcgen05.mma kind::mxf8f6f4 with block scaling multiplies each
// 32-wide K step of a row of A (and of B) by its UE8M0 scale and accumulates
// in fp32 TMEM across the whole K range, so no CUDA-core promotion is left.
// A scale of the 1x128 / 128x128 scheme covers four such K steps: all four
// MMAs of one 128-wide K block read the same scale byte.  The result equals
// the fine-grained-scaled GEMM of the same inputs up to the order of fp32
// accumulation.
//
// B200 design of one CTA (one per SM, persistent over 128 x BN tiles):
//   warp 4 (A producer) : per stage of KS K blocks, one 3-D TMA box of A;
//   warp 5 (B producer) : the same for B (each TMA instruction costs its
//                         issuing warp a roughly fixed time, so A and B are
//                         issued by different warps);
//   warp 6 (scale loader): copies the packed scale words of the tile's 128
//                         rows of A and BN rows of B, one K-block group at a
//                         time, into a 4-slot staging ring (cp.async, in the
//                         order tcgen05.cp wants: 32 rows of 16 bytes, row r
//                         holding rows r, r+32, r+64, r+96);
//   warp 8 (scale writer): per stage, copies the stage's group from the
//                         ring into the stage and fences it for the async
//                         proxy (a separate warp, so that no global load is
//                         in flight when it releases the stage);
//   warp 7 (MMA)        : copies the stage's scale chunks into TMEM
//                         (tcgen05.cp 32x128b.warpx4, replicated over the
//                         four lane quarters), issues 4 block-scaled MMAs per
//                         K block into one of two TMEM accumulators, and
//                         commits to free the stage / hand over the tile;
//   warps 0-3 (epilogue): read the finished accumulator from TMEM (thread t =
//                         tile row t), free it, round to bf16 and TMA-store
//                         64-column boxes (row by row where a grouped layout
//                         must leave rows untouched).
// The next tile's MMAs run in the other accumulator under the epilogue.
//
// Waits are bounded as in the fine-grained kernel: a wait that runs out
// records DG_ERR_TIMEOUT, raises the CTA's abort flag and every role leaves;
// copies and MMAs in flight are drained and TMEM freed before exit.
#pragma once

#include "fp8_gemm_kernel.cuh"
#include "fp8_gemm_pair_kernel.cuh"

namespace dg {

// The scale loader's copy of one K-block group (four K blocks): lane r
// copies the packed words of rows r, r+32, r+64, r+96 of the tile's 128 rows
// of A and of each 128-row chunk of its BN rows of B into a staging slot of
// shared memory, already in the order tcgen05.cp wants (row r of a chunk =
// 16 bytes at 16 r), with cp.async, and each lane's copies arrive on the
// slot's barrier when they land (so the loader never waits for them).  Rows
// past the matrix are zero-filled (their operand rows are zero too).
template <int CHUNKS>
__device__ __forceinline__ void sf_load_group(uint32_t slot, uint32_t staged_bar, const int32_t *sfa_g,
                                              const int32_t *sfb_g, const GemmParams &p, int a_row0, int n_row0,
                                              int kg)
{
    const int32_t *sa = sfa_g + static_cast<size_t>(kg) * p.sfa_ld;
    const int32_t *sb = sfb_g + static_cast<size_t>(kg) * p.nbn;
    const uint32_t dst = slot + 16 * (threadIdx.x % 32);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int r = a_row0 + 32 * j;
        cp_async_4_zfill(dst + 4 * j, r < p.M ? static_cast<const void *>(sa + r) : static_cast<const void *>(sa),
                         r < p.M ? 4u : 0u);
    }
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n_row0 + 128 * c + 32 * j;
            cp_async_4_zfill(dst + 512 * (1 + c) + 4 * j,
                             n < p.N ? static_cast<const void *>(sb + n / 128) : static_cast<const void *>(sb),
                             n < p.N ? 4u : 0u);
        }
    }
    cp_async_mbar_arrive_noinc(staged_bar);
}

// Copies this lane's rows of a staged group into a pipeline stage.
template <int CHUNKS>
__device__ __forceinline__ void sf_copy_rows(uint32_t dst_stage, uint32_t src_slot)
{
    const uint32_t off = 16 * (threadIdx.x % 32);
#pragma unroll
    for (int c = 0; c < 1 + CHUNKS; ++c)
        st_shared_v4(dst_stage + 512 * c + off, ld_shared_v4u(src_slot + 512 * c + off));
}

// BN: tile width; STAGES: ring depth; KS: 128-wide K blocks per stage (1, 2
// or 4, so a stage never straddles a word of four packed K-block scales).
template <int BN_, int STAGES_, int KS_>
struct BsConfig {
    static constexpr int BN = BN_;
    static constexpr int STAGES = STAGES_;
    static constexpr int KS = KS_;
    static constexpr int NUM_EPI_WARPS = 4;
    static constexpr int PRODUCER_A = 4;
    static constexpr int PRODUCER_B = 5;
    static constexpr int SF_LOADER = 6;
    static constexpr int MMA_WARP = 7;
    static constexpr int SF_WRITER = 8;
    static constexpr int THREADS = 288;
    static constexpr int A_BYTES = kBM * kBK;
    static constexpr int B_BYTES = BN * kBK;
    static constexpr int STAGE_A = KS * A_BYTES;
    static constexpr int STAGE_B = KS * B_BYTES;
    // scale chunks: one of 128 rows per 128 tile rows (A: 1, B: ceil(BN/128))
    static constexpr int SFB_CHUNKS = (BN + 127) / 128;
    static constexpr int SF_STAGE_BYTES = 512 * (1 + SFB_CHUNKS);
    // TMEM: two fp32 accumulators, then two scale slots (A: 4 columns, B: 4
    // per chunk) used by alternate stages.
    static constexpr int ACC_STRIDE = (BN + 31) / 32 * 32;
    static constexpr int NACC = 2;
    static constexpr int SF_COL0 = NACC * ACC_STRIDE;
    static constexpr int SF_SLOT_COLS = 16;
    static constexpr int TMEM_COLS = SF_COL0 + 2 * SF_SLOT_COLS <= 256 ? 256 : 512;
    static constexpr int SF_RING = 4;  // staging slots between the scale loader and writer
    static constexpr int BAR_BYTES = 8 * (2 * STAGES + 2 * NACC + 2 * SF_RING) + 16;
    // epilogue boxes: 64 columns x 128 rows with 128-byte swizzle, plus a
    // remainder box (unswizzled)
    static constexpr int EPI_FULL_BOXES = BN / 64;
    static constexpr int EPI_REM = BN % 64;
    static constexpr int EPI_BOXES = EPI_FULL_BOXES + (EPI_REM > 0 ? 1 : 0);
    static constexpr int EPI_BOX_BYTES = kBM * 128;
    static constexpr int PIPE_BYTES = STAGES * (STAGE_A + STAGE_B + SF_STAGE_BYTES) + SF_RING * SF_STAGE_BYTES;
    static constexpr int EPI_OFFSET = (PIPE_BYTES + BAR_BYTES + 1023) / 1024 * 1024;
    static constexpr int EPI_BUFS = 1024 + EPI_OFFSET + 2 * EPI_BOX_BYTES <= 232448 ? 2 : 1;
    static constexpr int SMEM_BYTES = 1024 + EPI_OFFSET + EPI_BUFS * EPI_BOX_BYTES;

    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128: multiple of 16, <= 256");
    static_assert(EPI_REM % 8 == 0, "remainder box must be whole 16-byte chunks");
    static_assert(KS == 1 || KS == 2 || KS == 4, "a stage must lie inside one word of packed scales");
    static_assert(SF_COL0 % 16 == 0, "scale slots start on a 16-column boundary");
    static_assert(SF_COL0 + 2 * SF_SLOT_COLS <= 512, "accumulators and scale slots must fit in TMEM");
    static_assert(4 + 4 * SFB_CHUNKS <= SF_SLOT_COLS, "scale slot too small");
    static_assert(B_BYTES % 1024 == 0, "B tiles must keep 1024-byte swizzle atoms aligned");
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

template <int BN, int STAGES, int KS, int LAYOUT>
__global__ void __launch_bounds__(BsConfig<BN, STAGES, KS>::THREADS, 1)
    fp8_gemm_bs_kernel(const __grid_constant__ CUtensorMap tmap_a,
                       const __grid_constant__ CUtensorMap tmap_b,
                       const __grid_constant__ CUtensorMap tmap_d64,
                       const __grid_constant__ CUtensorMap tmap_drem, const GemmParams p)
{
    using Cfg = BsConfig<BN, STAGES, KS>;
    static_assert(LAYOUT == kDense || LAYOUT == kContiguous || LAYOUT == kMasked,
                  "block-scaled mode: dense, contiguous and masked layouts");
    constexpr int NACC = Cfg::NACC;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *a_tiles = smem;                                  // [STAGES][KS][128][128 B]
    uint8_t *b_tiles = smem + STAGES * Cfg::STAGE_A;          // [STAGES][KS][BN][128 B]
    uint8_t *sf_tiles = b_tiles + STAGES * Cfg::STAGE_B;      // [STAGES][1+SFB_CHUNKS][32][16 B]
    uint8_t *sf_ring = sf_tiles + STAGES * Cfg::SF_STAGE_BYTES;  // [SF_RING][1+SFB_CHUNKS][32][16 B]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sf_ring + Cfg::SF_RING * Cfg::SF_STAGE_BYTES);
    uint64_t *full_bar = bars;                    // A box, B box and scales of the stage landed
    uint64_t *empty_bar = bars + STAGES;          // MMAs (and scale copies) of the stage done
    uint64_t *tfull_bar = bars + 2 * STAGES;      // accumulator holds a finished tile
    uint64_t *tempty_bar = bars + 2 * STAGES + NACC;  // accumulator read out
    uint64_t *staged_full = bars + 2 * STAGES + 2 * NACC;           // a staging slot holds its group
    uint64_t *staged_empty = bars + 2 * STAGES + 2 * NACC + Cfg::SF_RING;  // the writer is done with it
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 2 * NACC + 2 * Cfg::SF_RING);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    uint8_t *epi_stage = smem + Cfg::EPI_OFFSET;

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    if (warp == Cfg::PRODUCER_A && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            // full: two expect-tx arrivals (A, B) and the scale warp's arrival
            mbar_init(smem_addr(full_bar + s), 3);
            mbar_init(smem_addr(empty_bar + s), 1);
        }
        for (int b = 0; b < NACC; ++b) {
            mbar_init(smem_addr(tfull_bar + b), 1);
            mbar_init(smem_addr(tempty_bar + b), Cfg::NUM_EPI_WARPS);
        }
        for (int r = 0; r < Cfg::SF_RING; ++r) {
            mbar_init(smem_addr(staged_full + r), 32);  // one cp.async arrival per loader lane
            mbar_init(smem_addr(staged_empty + r), 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmap_a);
        tma_prefetch_desc(&tmap_b);
        if (Cfg::EPI_FULL_BOXES > 0)
            tma_prefetch_desc(&tmap_d64);
        if (Cfg::EPI_REM > 0)
            tma_prefetch_desc(&tmap_drem);
    }
    if (warp == Cfg::MMA_WARP) {
        tmem_alloc(smem_addr(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish_alloc_permit();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    const uint64_t tmo = p.timeout_ns;
    const uint64_t drain_tmo = tmo > 1000000000ull ? tmo : 1000000000ull;

    if (warp == Cfg::PRODUCER_A || warp == Cfg::PRODUCER_B) {
        // ------------------------------------------------- TMA producers
        const bool is_a = warp == Cfg::PRODUCER_A;
        TileScheduler<LAYOUT> sched(p);
        TileCoord tc;
        uint32_t stage = 0, phase = 0, issued = 0;
        bool ok = !(p.stall_injection && blockIdx.x == 0);
        while (ok && sched.next(tc, is_a && lane == 0)) {
            const int row = is_a ? (LAYOUT == kMasked ? tc.g * p.M : 0) + tc.mb * kBM
                                 : tc.g * p.N + tc.nb * BN;
            for (int kb0 = 0; kb0 < p.num_kb; kb0 += KS) {
                if (!warp_wait_bounded(smem_addr(empty_bar + stage), phase ^ 1, tmo, abort_flag,
                                       kRoleProducer, stage)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = smem_addr(full_bar + stage);
                if (elect_one()) {
                    if (is_a) {
                        mbar_arrive_expect_tx(fb, Cfg::STAGE_A);
                        tma_load_3d(smem_addr(a_tiles + stage * Cfg::STAGE_A), &tmap_a, fb, 0, row, kb0);
                    } else {
                        mbar_arrive_expect_tx(fb, Cfg::STAGE_B);
                        tma_load_3d(smem_addr(b_tiles + stage * Cfg::STAGE_B), &tmap_b, fb, 0, row, kb0);
                    }
                }
                __syncwarp();
                ++issued;
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        // the copies of the last min(STAGES, issued) stages land before exit
        if (lane == 0) {
            const uint32_t first = issued > STAGES ? issued - STAGES : 0;
            for (uint32_t i = first; i < issued; ++i)
                wait_bounded(smem_addr(full_bar + i % STAGES), (i / STAGES) & 1, drain_tmo, abort_flag,
                             kRoleDrain, i % STAGES, false);
        }
        __syncwarp();
    } else if (warp == Cfg::SF_LOADER) {
        // ------------------------------------------------- scale loader
        // Copies each K-block group's scale words into the staging ring as
        // soon as a slot is free, running up to SF_RING groups ahead.
        TileScheduler<LAYOUT> sched(p);
        TileCoord tc;
        uint32_t gs = 0;  // group sequence number over all tiles
        bool ok = true;
        while (ok && sched.next(tc, false)) {
            const int32_t *sfa_g =
                p.sfa + (LAYOUT == kMasked ? static_cast<size_t>(tc.g) * p.num_kg * p.sfa_ld : 0);
            const int32_t *sfb_g = p.sfb + static_cast<size_t>(tc.g) * p.num_kg * p.nbn;
            const int a_row0 = tc.mb * kBM + lane;
            const int n_row0 = tc.nb * BN + lane;
            for (int kg = 0; kg < p.num_kg; ++kg, ++gs) {
                const uint32_t slot = gs % Cfg::SF_RING, sph = (gs / Cfg::SF_RING) & 1;
                if (!warp_wait_bounded(smem_addr(staged_empty + slot), sph ^ 1, tmo, abort_flag, kRoleProducer, 96 + slot)) {
                    ok = false;
                    break;
                }
                sf_load_group<Cfg::SFB_CHUNKS>(smem_addr(sf_ring + slot * Cfg::SF_STAGE_BYTES),
                                               smem_addr(staged_full + slot), sfa_g, sfb_g, p, a_row0, n_row0, kg);
            }
        }
        cp_async_wait_all();  // no copy still in flight at exit
    } else if (warp == Cfg::SF_WRITER) {
        // ------------------------------------------------- scale writer
        // Per stage: the stage's group from the staging ring into the
        // stage's scale chunk, fenced for the async proxy (tcgen05.cp reads
        // it), then the arrival on the full barrier.  This warp has no
        // global memory operations in flight, so its release is cheap.
        TileScheduler<LAYOUT> sched(p);
        TileCoord tc;
        uint32_t stage = 0, phase = 0, gs = 0;
        bool ok = true;
        while (ok && sched.next(tc, false)) {
            for (int kb0 = 0; kb0 < p.num_kb; kb0 += KS) {
                const uint32_t g = gs + static_cast<uint32_t>(kb0 / 4);
                const uint32_t slot = g % Cfg::SF_RING, sph = (g / Cfg::SF_RING) & 1;
                if ((kb0 % 4 == 0 && !warp_wait_bounded(smem_addr(staged_full + slot), sph, tmo, abort_flag, kRoleProducer, 112 + slot)) ||
                    !warp_wait_bounded(smem_addr(empty_bar + stage), phase ^ 1, tmo, abort_flag, kRoleProducer, 32 + stage)) {
                    ok = false;
                    break;
                }
                sf_copy_rows<Cfg::SFB_CHUNKS>(smem_addr(sf_tiles + stage * Cfg::SF_STAGE_BYTES),
                                              smem_addr(sf_ring + slot * Cfg::SF_STAGE_BYTES));
                // generic-proxy writes, read next by tcgen05.cp (async proxy)
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(smem_addr(full_bar + stage));
                    // the group's last stage: its staging slot may be refilled
                    if (kb0 + KS >= p.num_kb || (kb0 + KS) % 4 == 0)
                        mbar_arrive(smem_addr(staged_empty + slot));
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            gs += static_cast<uint32_t>(p.num_kg);
        }
    } else if (warp == Cfg::MMA_WARP) {
        // ------------------------------------------------------ MMA issuer
        TileScheduler<LAYOUT> sched(p);
        TileCoord tc;
        uint32_t stage = 0, phase = 0, acc_i = 0, stage_i = 0;
        uint32_t last_bar = 0, last_parity = 0;
        bool ok = true;
        const uint64_t a_desc0 = smem_desc_k_sw128(smem_addr(a_tiles));
        const uint64_t b_desc0 = smem_desc_k_sw128(smem_addr(b_tiles));
        const uint64_t sf_desc0 = smem_desc_sf_chunk(smem_addr(sf_tiles));
        while (ok && sched.next(tc, false)) {
            const uint32_t buf = acc_i % NACC, tph = (acc_i / NACC) & 1;
            if (!warp_wait_bounded(smem_addr(tempty_bar + buf), tph ^ 1, tmo, abort_flag, kRoleMma,
                                   16 + buf)) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            const uint32_t d_tmem = tmem_base + buf * Cfg::ACC_STRIDE;
            for (int kb0 = 0; kb0 < p.num_kb; kb0 += KS) {
                if (!warp_wait_bounded(smem_addr(full_bar + stage), phase, tmo, abort_flag, kRoleMma,
                                       stage)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t sf_col = tmem_base + Cfg::SF_COL0 + (stage_i & 1) * Cfg::SF_SLOT_COLS;
                if (elect_one()) {
                    const uint64_t sfd = sf_desc0 + static_cast<uint64_t>((stage * Cfg::SF_STAGE_BYTES) >> 4);
#pragma unroll
                    for (int c = 0; c < 1 + Cfg::SFB_CHUNKS; ++c)
                        tmem_cp_32x128b_warpx4(sf_col + 4 * c, sfd + static_cast<uint64_t>((512 * c) >> 4));
#pragma unroll
                    for (int q = 0; q < KS; ++q) {
                        const int kb = kb0 + q;
                        if (kb >= p.num_kb)
                            break;
                        const uint32_t byte = static_cast<uint32_t>(kb & 3);
                        const uint32_t idesc = idesc_mxf8_e4m3_ue8m0(kBM, BN, byte);
                        const uint64_t ad = a_desc0 + static_cast<uint64_t>((stage * Cfg::STAGE_A + q * Cfg::A_BYTES) >> 4);
                        const uint64_t bd = b_desc0 + static_cast<uint64_t>((stage * Cfg::STAGE_B + q * Cfg::B_BYTES) >> 4);
#pragma unroll
                        for (int j = 0; j < kBK / 32; ++j)
                            mma_mxf8f6f4_bs(d_tmem, ad + 2 * j, bd + 2 * j, idesc, sf_col | (byte << 30),
                                            (sf_col + 4) | (byte << 30), (kb > 0 || j > 0) ? 1u : 0u);
                    }
                    mma_commit(smem_addr(empty_bar + stage));
                }
                __syncwarp();
                last_bar = smem_addr(empty_bar + stage);
                last_parity = phase;
                ++stage_i;
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (!ok)
                break;
            if (elect_one())
                mma_commit(smem_addr(tfull_bar + buf));
            __syncwarp();
            last_bar = smem_addr(tfull_bar + buf);
            last_parity = tph;
            ++acc_i;
        }
        if (lane == 0 && last_bar != 0)
            wait_bounded(last_bar, last_parity, drain_tmo, abort_flag, kRoleDrain, 32, false);
        __syncwarp();
    } else {
        // ------------------------------------------------------- epilogue
        const int quad = warp;             // TMEM lane quarter of this warp
        const int row = quad * 32 + lane;  // tile row == TMEM lane
        const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
        TileScheduler<LAYOUT> sched(p);
        TileCoord tc;
        uint32_t acc_i = 0;
        bool ok = true;
        while (ok && sched.next(tc, false)) {
            const uint32_t buf = acc_i % NACC, tph = (acc_i / NACC) & 1;
            ok = warp_wait_bounded(smem_addr(tfull_bar + buf), tph, tmo, abort_flag, kRolePromote, 16 + buf);
            // a warp that gave up takes the others with it (no warp may be
            // left waiting at a later named barrier)
            if (!named_barrier_and(1, 128, ok)) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            const int m_local = tc.mb * kBM + row;
            bool row_ok;
            if constexpr (LAYOUT == kDense) {
                row_ok = m_local < p.M;
            } else if constexpr (LAYOUT == kContiguous) {
                row_ok = false;
                if (m_local < p.M) {
                    const int idx = __ldg(p.m_indices + m_local);
                    row_ok = idx == tc.g;
                    if (idx >= 0 && idx != tc.g)
                        record_status(kCodeBadGroup, kRolePromote, 1);
                }
            } else {
                int mm = __ldg(p.masked_m + tc.g);
                mm = mm < 0 ? 0 : (mm > p.M ? p.M : mm);
                row_ok = m_local < mm;
            }
            const bool tile_rows_ok =
                named_barrier_and(1, 128, LAYOUT == kDense ? (tc.mb * kBM < p.M) : row_ok);
            const int grow0 = (LAYOUT == kMasked ? tc.g * p.M : 0) + tc.mb * kBM;
            const int col0 = tc.nb * BN;
            const uint32_t taddr = tmem_base + lane_bits + buf * Cfg::ACC_STRIDE;
#pragma unroll
            for (int bx = 0; bx < Cfg::EPI_BOXES; ++bx) {
                const bool full = bx < Cfg::EPI_FULL_BOXES;
                const int cbase = bx * 64;
                const int ncols = full ? 64 : Cfg::EPI_REM;
                uint32_t r[64];
                if (full)
                    tmem_load_cols<64>(taddr + cbase, r);
                else
                    tmem_load_cols<(Cfg::EPI_REM > 0 ? Cfg::EPI_REM : 8)>(taddr + cbase, r);
                tmem_ld_wait();
                float v[64];
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    v[i] = __uint_as_float(r[i]);
                if (bx == Cfg::EPI_BOXES - 1) {
                    // the whole accumulator is in registers: hand it back
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(smem_addr(tempty_bar + buf));
                }
                const bool box_in = col0 + cbase < p.N;
                if (tile_rows_ok) {
                    if (!box_in)
                        continue;  // uniform over the warpgroup
                    const uint32_t stg = smem_addr(epi_stage + (bx % Cfg::EPI_BUFS) * Cfg::EPI_BOX_BYTES);
                    if (threadIdx.x == 0)
                        bulk_wait_group_read<Cfg::EPI_BUFS - 1>();
                    named_barrier_sync(1, 128);
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        if (ch * 8 < ncols) {
                            const uint32_t off =
                                full ? static_cast<uint32_t>(row * 128 + ((ch ^ (row & 7)) * 16))
                                     : static_cast<uint32_t>(row * ncols * 2 + ch * 16);
                            st_shared_v4(stg + off, pack_bf16x8(v + ch * 8));
                        }
                    }
                    fence_proxy_async_smem();
                    named_barrier_sync(1, 128);
                    if (threadIdx.x == 0) {
                        tma_store_2d(full ? static_cast<const void *>(&tmap_d64)
                                          : static_cast<const void *>(&tmap_drem),
                                     stg, col0 + cbase, grow0);
                        bulk_commit_group();
                    }
                } else if (row_ok && box_in) {
                    const size_t grow = static_cast<size_t>(grow0) + row;
                    __nv_bfloat16 *drow = p.D + grow * p.N + col0 + cbase;
#pragma unroll
                    for (int c = 0; c < 64; c += 8)
                        if (c < ncols && col0 + cbase + c < p.N)
                            *reinterpret_cast<uint4 *>(drow + c) = pack_bf16x8(v + c);
                }
            }
            ++acc_i;
        }
        if (threadIdx.x == 0)
            bulk_wait_group<0>();
        __syncwarp();
    }

    __syncthreads();
    if (warp == Cfg::MMA_WARP) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

// ------------------------------------------------------------ CTA pairs
//
// The block-scaled mode on 256 x BN tiles shared by the two CTAs of a
// cluster (tcgen05 cta_group::2).  Per SM and K block the operand bytes drop
// from (128 + BN) * 128 to (128 + BN/2) * 128, which keeps the L2 -> SM feed
// below what the tensor cores consume at full rate.  Per CTA:
//   warp 4 / 5 : TMA boxes of its own 128 rows of A / BN/2 rows of B
//                (cta_group::2 loads signalling the leader's full barrier;
//                the leader's warps post the bytes of both CTAs);
//   warps 6, 8 : the scale words of its own 128 rows of A and of all BN rows
//                of B: the loader stages them (cp.async, a 4-slot ring), the
//                writer copies each stage's group into the stage, fences it
//                for the async proxy and announces it to the leader's full
//                barrier with a cluster-scope release (cheap, since the
//                writer has no global load in flight);
//   warp 7     : (leader only) tcgen05.cp.cta_group::2 of both CTAs' scale
//                chunks into their TMEM (a slot per stage), then the pair
//                MMAs; commits arrive on both CTAs' barriers (multicast
//                arrive, not a data copy);
//   warps 0-3  : the epilogue of its own 128 rows; the accumulator goes back
//                to the leader's MMA warp when both CTAs have read it.
// Every wait is bounded; a CTA that gives up raises its peer's abort flag.
template <int BN_, int STAGES_, int KS_>
struct BsPairConfig {
    static constexpr int BN = BN_;
    static constexpr int BN_HALF = BN / 2;
    static constexpr int STAGES = STAGES_;
    static constexpr int KS = KS_;
    static constexpr int NUM_EPI_WARPS = 4;
    static constexpr int PRODUCER_A = 4;
    static constexpr int PRODUCER_B = 5;
    static constexpr int SF_LOADER = 6;
    static constexpr int MMA_WARP = 7;
    static constexpr int SF_WRITER = 8;
    static constexpr int THREADS = 288;
    static constexpr int A_BYTES = kBM * kBK;
    static constexpr int B_BYTES = BN_HALF * kBK;
    static constexpr int STAGE_A = KS * A_BYTES;
    static constexpr int STAGE_B = KS * B_BYTES;
    static constexpr int SFB_CHUNKS = (BN + 127) / 128;
    static constexpr int SF_STAGE_BYTES = 512 * (1 + SFB_CHUNKS);
    static constexpr int ACC_STRIDE = (BN + 31) / 32 * 32;
    static constexpr int NACC = 2;
    static constexpr int SF_COL0 = NACC * ACC_STRIDE;
    static constexpr int SF_SLOT_COLS = 16;  // one slot per stage
    static constexpr int TMEM_COLS = 512;
    static constexpr int SF_RING = 4;  // staging slots between the scale loader and writer
    static constexpr int BAR_BYTES = 8 * (2 * STAGES + 2 * NACC + 2 * SF_RING) + 16;
    static constexpr int EPI_FULL_BOXES = BN / 64;
    static constexpr int EPI_REM = BN % 64;
    static constexpr int EPI_BOXES = EPI_FULL_BOXES + (EPI_REM > 0 ? 1 : 0);
    static constexpr int EPI_BOX_BYTES = kBM * 128;
    static constexpr int PIPE_BYTES = STAGES * (STAGE_A + STAGE_B + SF_STAGE_BYTES) + SF_RING * SF_STAGE_BYTES;
    static constexpr int EPI_OFFSET = (PIPE_BYTES + BAR_BYTES + 1023) / 1024 * 1024;
    static constexpr int EPI_BUFS = 1024 + EPI_OFFSET + 2 * EPI_BOX_BYTES <= 232448 ? 2 : 1;
    static constexpr int SMEM_BYTES = 1024 + EPI_OFFSET + EPI_BUFS * EPI_BOX_BYTES;

    static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "pair MMA N (M = 256)");
    static_assert(EPI_REM % 8 == 0, "remainder box must be whole 16-byte chunks");
    static_assert(KS == 1 || KS == 2 || KS == 4, "a stage must lie inside one word of packed scales");
    static_assert(SF_COL0 % 16 == 0 && SF_COL0 + STAGES * SF_SLOT_COLS <= TMEM_COLS,
                  "accumulators and per-stage scale slots must fit in TMEM");
    static_assert(4 + 4 * SFB_CHUNKS <= SF_SLOT_COLS, "scale slot too small");
    static_assert(B_BYTES % 1024 == 0, "B tiles must keep 1024-byte swizzle atoms aligned");
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

// Bounded pair wait whose successful acquire is at cluster scope (the phase
// includes a release arrival from the peer CTA).
__device__ __forceinline__ bool pair_warp_wait_acq_cluster(uint32_t bar, uint32_t parity, uint64_t timeout_ns,
                                                           volatile int *abort_flag, uint32_t peer_abort,
                                                           uint32_t role, uint32_t stage)
{
    int ok = 0;
    if ((threadIdx.x & 31) == 0) {
        ok = 1;
        if (!mbar_try_wait_acq_cluster(bar, parity)) {
            const uint64_t t0 = global_timer_ns();
            uint32_t spins = 0;
            while (!mbar_try_wait_acq_cluster(bar, parity)) {
                if ((++spins & 63u) == 0) {
                    if (*abort_flag) {
                        ok = 0;
                        break;
                    }
                    if (global_timer_ns() - t0 > timeout_ns) {
                        *abort_flag = 1;
                        record_status(kCodeTimeout, role, stage);
                        ok = 0;
                        break;
                    }
                }
            }
        }
        if (!ok)
            st_shared_cluster_u32(peer_abort, 1u);
    }
    return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

template <int BN, int STAGES, int KS, int LAYOUT>
__global__ void __launch_bounds__(BsPairConfig<BN, STAGES, KS>::THREADS, 1)
    fp8_gemm_bs_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                            const __grid_constant__ CUtensorMap tmap_b,
                            const __grid_constant__ CUtensorMap tmap_d64,
                            const __grid_constant__ CUtensorMap tmap_drem, const GemmParams p)
{
    using Cfg = BsPairConfig<BN, STAGES, KS>;
    static_assert(LAYOUT == kDense || LAYOUT == kContiguous || LAYOUT == kMasked,
                  "block-scaled mode: dense, contiguous and masked layouts");
    constexpr int NACC = Cfg::NACC;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *a_tiles = smem;                              // [STAGES][KS][128][128 B]
    uint8_t *b_tiles = smem + STAGES * Cfg::STAGE_A;      // [STAGES][KS][BN/2][128 B]
    uint8_t *sf_tiles = b_tiles + STAGES * Cfg::STAGE_B;  // [STAGES][1+SFB_CHUNKS][32][16 B]
    uint8_t *sf_ring = sf_tiles + STAGES * Cfg::SF_STAGE_BYTES;  // [SF_RING][1+SFB_CHUNKS][32][16 B]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sf_ring + Cfg::SF_RING * Cfg::SF_STAGE_BYTES);
    uint64_t *full_bar = bars;                        // (leader) both CTAs' boxes and scales landed
    uint64_t *empty_bar = bars + STAGES;              // pair MMAs and scale copies of the stage done
    uint64_t *tfull_bar = bars + 2 * STAGES;          // accumulator holds a finished tile
    uint64_t *tempty_bar = bars + 2 * STAGES + NACC;  // (leader) both CTAs read the accumulator
    uint64_t *staged_full = bars + 2 * STAGES + 2 * NACC;           // a staging slot holds its group
    uint64_t *staged_empty = bars + 2 * STAGES + 2 * NACC + Cfg::SF_RING;  // the writer is done with it
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 2 * NACC + 2 * Cfg::SF_RING);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    uint8_t *epi_stage = smem + Cfg::EPI_OFFSET;

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (warp == Cfg::PRODUCER_A && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            // full: the leader's two expect-tx arrivals and both CTAs' scale
            // warps
            mbar_init(smem_addr(full_bar + s), 4);
            mbar_init(smem_addr(empty_bar + s), 1);
        }
        for (int b = 0; b < NACC; ++b) {
            mbar_init(smem_addr(tfull_bar + b), 1);
            mbar_init(smem_addr(tempty_bar + b), 2 * Cfg::NUM_EPI_WARPS);
        }
        for (int r = 0; r < Cfg::SF_RING; ++r) {
            mbar_init(smem_addr(staged_full + r), 32);  // one cp.async arrival per loader lane
            mbar_init(smem_addr(staged_empty + r), 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmap_a);
        tma_prefetch_desc(&tmap_b);
        if (Cfg::EPI_FULL_BOXES > 0)
            tma_prefetch_desc(&tmap_d64);
        if (Cfg::EPI_REM > 0)
            tma_prefetch_desc(&tmap_drem);
    }
    if (warp == Cfg::MMA_WARP) {
        tmem_alloc_pair(smem_addr(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish_alloc_permit_pair();
    }
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before either signals the other
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    const uint64_t tmo = p.timeout_ns;
    const uint64_t drain_tmo = tmo > 1000000000ull ? tmo : 1000000000ull;
    const uint32_t peer_abort = map_shared_rank(smem_addr(const_cast<int *>(abort_flag)), rank ^ 1u);
    const uint32_t full_leader = map_shared_rank(smem_addr(full_bar), 0);
    const uint32_t tempty_leader = map_shared_rank(smem_addr(tempty_bar), 0);

    if (warp == Cfg::PRODUCER_A || warp == Cfg::PRODUCER_B) {
        // ------------------------------------------------- TMA producers
        const bool is_a = warp == Cfg::PRODUCER_A;
        PairScheduler<LAYOUT> sched(p);
        TileCoord tc;
        uint32_t stage = 0, phase = 0;
        bool ok = !(p.stall_injection && blockIdx.x < 2);
        while (ok && sched.next(tc, is_a && leader && lane == 0)) {
            const int row = is_a ? (LAYOUT == kMasked ? tc.g * p.M : 0) + tc.mb * kPairBM +
                                       static_cast<int>(rank) * kBM
                                 : tc.g * p.N + tc.nb * BN + static_cast<int>(rank) * Cfg::BN_HALF;
            for (int kb0 = 0; kb0 < p.num_kb; kb0 += KS) {
                if (!pair_warp_wait(smem_addr(empty_bar + stage), phase ^ 1, tmo, abort_flag, peer_abort,
                                    kRoleProducer, stage)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = full_leader + 8 * stage;
                if (elect_one()) {
                    if (is_a) {
                        if (leader)
                            mbar_arrive_expect_tx(smem_addr(full_bar + stage), 2 * Cfg::STAGE_A);
                        tma_load_3d_pair(smem_addr(a_tiles + stage * Cfg::STAGE_A), &tmap_a, fb, 0, row, kb0);
                    } else {
                        if (leader)
                            mbar_arrive_expect_tx(smem_addr(full_bar + stage), 2 * Cfg::STAGE_B);
                        tma_load_3d_pair(smem_addr(b_tiles + stage * Cfg::STAGE_B), &tmap_b, fb, 0, row, kb0);
                    }
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        // On the normal path every box has landed (the leader's MMA waited
        // for it).  After an abort, boxes may still be in flight towards a
        // barrier or tile of either CTA: give them a bounded moment to land
        // before the pair passes the exit barrier.
        if (!ok && lane == 0) {
            const uint64_t t0 = global_timer_ns();
            while (global_timer_ns() - t0 < 200000ull) {
            }
        }
        __syncwarp();
    } else if (warp == Cfg::SF_LOADER) {
        // ------------------------------------------------- scale loader
        // Copies each K-block group's scale words into the staging ring as
        // soon as a slot is free, running up to SF_RING groups ahead.
        PairScheduler<LAYOUT> sched(p);
        TileCoord tc;
        uint32_t gs = 0;  // group sequence number over all tiles
        bool ok = true;
        while (ok && sched.next(tc, false)) {
            const int32_t *sfa_g =
                p.sfa + (LAYOUT == kMasked ? static_cast<size_t>(tc.g) * p.num_kg * p.sfa_ld : 0);
            const int32_t *sfb_g = p.sfb + static_cast<size_t>(tc.g) * p.num_kg * p.nbn;
            const int a_row0 = tc.mb * kPairBM + static_cast<int>(rank) * kBM + lane;
            const int n_row0 = tc.nb * BN + lane;
            for (int kg = 0; kg < p.num_kg; ++kg, ++gs) {
                const uint32_t slot = gs % Cfg::SF_RING, sph = (gs / Cfg::SF_RING) & 1;
                if (!pair_warp_wait(smem_addr(staged_empty + slot), sph ^ 1, tmo, abort_flag, peer_abort, kRoleProducer, 96 + slot)) {
                    ok = false;
                    break;
                }
                sf_load_group<Cfg::SFB_CHUNKS>(smem_addr(sf_ring + slot * Cfg::SF_STAGE_BYTES),
                                               smem_addr(staged_full + slot), sfa_g, sfb_g, p, a_row0, n_row0, kg);
            }
        }
        cp_async_wait_all();  // no copy still in flight at exit
    } else if (warp == Cfg::SF_WRITER) {
        // ------------------------------------------------- scale writer
        // Per stage: the stage's group from the staging ring into the
        // stage's scale chunk, fenced for the async proxy (tcgen05.cp reads
        // it), then the arrival on the full barrier.  This warp has no
        // global memory operations in flight, so its release is cheap.
        PairScheduler<LAYOUT> sched(p);
        TileCoord tc;
        uint32_t stage = 0, phase = 0, gs = 0;
        bool ok = true;
        while (ok && sched.next(tc, false)) {
            for (int kb0 = 0; kb0 < p.num_kb; kb0 += KS) {
                const uint32_t g = gs + static_cast<uint32_t>(kb0 / 4);
                const uint32_t slot = g % Cfg::SF_RING, sph = (g / Cfg::SF_RING) & 1;
                if ((kb0 % 4 == 0 && !pair_warp_wait(smem_addr(staged_full + slot), sph, tmo, abort_flag, peer_abort, kRoleProducer, 112 + slot)) ||
                    !pair_warp_wait(smem_addr(empty_bar + stage), phase ^ 1, tmo, abort_flag, peer_abort, kRoleProducer, 32 + stage)) {
                    ok = false;
                    break;
                }
                sf_copy_rows<Cfg::SFB_CHUNKS>(smem_addr(sf_tiles + stage * Cfg::SF_STAGE_BYTES),
                                              smem_addr(sf_ring + slot * Cfg::SF_STAGE_BYTES));
                // generic-proxy writes, read next by tcgen05.cp (async proxy)
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_release_cluster(full_leader + 8 * stage);
                    // the group's last stage: its staging slot may be refilled
                    if (kb0 + KS >= p.num_kb || (kb0 + KS) % 4 == 0)
                        mbar_arrive(smem_addr(staged_empty + slot));
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            gs += static_cast<uint32_t>(p.num_kg);
        }
    } else if (warp == Cfg::MMA_WARP) {
        // ------------------------------------------------ MMA issuer (leader)
        if (leader) {
            PairScheduler<LAYOUT> sched(p);
            TileCoord tc;
            uint32_t stage = 0, phase = 0, acc_i = 0;
            uint32_t last_bar = 0, last_parity = 0;
            bool ok = true;
            const uint64_t a_desc0 = smem_desc_k_sw128(smem_addr(a_tiles));
            const uint64_t b_desc0 = smem_desc_k_sw128(smem_addr(b_tiles));
            const uint64_t sf_desc0 = smem_desc_sf_chunk(smem_addr(sf_tiles));
            while (ok && sched.next(tc, false)) {
                const uint32_t buf = acc_i % NACC, tph = (acc_i / NACC) & 1;
                if (!pair_warp_wait(smem_addr(tempty_bar + buf), tph ^ 1, tmo, abort_flag, peer_abort, kRoleMma,
                                    16 + buf)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + buf * Cfg::ACC_STRIDE;
                for (int kb0 = 0; kb0 < p.num_kb; kb0 += KS) {
                    if (!pair_warp_wait_acq_cluster(smem_addr(full_bar + stage), phase, tmo, abort_flag, peer_abort,
                                                    kRoleMma, stage)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t sf_col = tmem_base + Cfg::SF_COL0 + stage * Cfg::SF_SLOT_COLS;
                    if (elect_one()) {
                        const uint64_t sfd = sf_desc0 + static_cast<uint64_t>((stage * Cfg::SF_STAGE_BYTES) >> 4);
#pragma unroll
                        for (int c = 0; c < 1 + Cfg::SFB_CHUNKS; ++c)
                            tmem_cp_32x128b_warpx4_pair(sf_col + 4 * c, sfd + static_cast<uint64_t>((512 * c) >> 4));
#pragma unroll
                        for (int q = 0; q < KS; ++q) {
                            const int kb = kb0 + q;
                            if (kb >= p.num_kb)
                                break;
                            const uint32_t byte = static_cast<uint32_t>(kb & 3);
                            const uint32_t idesc = idesc_mxf8_e4m3_ue8m0(kPairBM, BN, byte);
                            const uint64_t ad =
                                a_desc0 + static_cast<uint64_t>((stage * Cfg::STAGE_A + q * Cfg::A_BYTES) >> 4);
                            const uint64_t bd =
                                b_desc0 + static_cast<uint64_t>((stage * Cfg::STAGE_B + q * Cfg::B_BYTES) >> 4);
#pragma unroll
                            for (int j = 0; j < kBK / 32; ++j)
                                mma_mxf8f6f4_bs_pair(d_tmem, ad + 2 * j, bd + 2 * j, idesc, sf_col | (byte << 30),
                                                     (sf_col + 4) | (byte << 30), (kb > 0 || j > 0) ? 1u : 0u);
                        }
                        mma_commit_pair_multicast(smem_addr(empty_bar + stage), 0x3);
                    }
                    __syncwarp();
                    last_bar = smem_addr(empty_bar + stage);
                    last_parity = phase;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok)
                    break;
                if (elect_one())
                    mma_commit_pair_multicast(smem_addr(tfull_bar + buf), 0x3);
                __syncwarp();
                last_bar = smem_addr(tfull_bar + buf);
                last_parity = tph;
                ++acc_i;
            }
            if (lane == 0 && last_bar != 0)
                wait_bounded(last_bar, last_parity, drain_tmo, abort_flag, kRoleDrain, 32, false);
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------- epilogue
        const int quad = warp;
        const int row = quad * 32 + lane;  // row within this CTA's half == TMEM lane
        const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
        PairScheduler<LAYOUT> sched(p);
        TileCoord tc;
        uint32_t acc_i = 0;
        bool ok = true;
        while (ok && sched.next(tc, false)) {
            const uint32_t buf = acc_i % NACC, tph = (acc_i / NACC) & 1;
            ok = pair_warp_wait(smem_addr(tfull_bar + buf), tph, tmo, abort_flag, peer_abort, kRolePromote,
                                16 + buf);
            if (!named_barrier_and(1, 128, ok)) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            const int m_half = tc.mb * kPairBM + static_cast<int>(rank) * kBM;
            const int m_local = m_half + row;
            bool row_ok;
            if constexpr (LAYOUT == kDense) {
                row_ok = m_local < p.M;
            } else if constexpr (LAYOUT == kContiguous) {
                row_ok = false;
                const int block_g = m_half < p.M ? __ldg(p.m_indices + m_half) : -1;
                if (m_local < p.M && block_g >= 0) {
                    const int idx = __ldg(p.m_indices + m_local);
                    row_ok = idx == tc.g;
                    if (idx >= 0 && idx != block_g)
                        record_status(kCodeBadGroup, kRolePromote, 1);
                }
            } else {
                int mm = __ldg(p.masked_m + tc.g);
                mm = mm < 0 ? 0 : (mm > p.M ? p.M : mm);
                row_ok = m_local < mm;
            }
            const bool tile_rows_ok = named_barrier_and(1, 128, LAYOUT == kDense ? (m_half < p.M) : row_ok);
            const int grow0 = (LAYOUT == kMasked ? tc.g * p.M : 0) + m_half;
            const int col0 = tc.nb * BN;
            const uint32_t taddr = tmem_base + lane_bits + buf * Cfg::ACC_STRIDE;
#pragma unroll
            for (int bx = 0; bx < Cfg::EPI_BOXES; ++bx) {
                const bool full = bx < Cfg::EPI_FULL_BOXES;
                const int cbase = bx * 64;
                const int ncols = full ? 64 : Cfg::EPI_REM;
                uint32_t r[64];
                if (full)
                    tmem_load_cols<64>(taddr + cbase, r);
                else
                    tmem_load_cols<(Cfg::EPI_REM > 0 ? Cfg::EPI_REM : 8)>(taddr + cbase, r);
                tmem_ld_wait();
                if (bx == Cfg::EPI_BOXES - 1) {
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive_cluster(tempty_leader + 8 * buf);
                }
                float v[64];
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    v[i] = __uint_as_float(r[i]);
                const bool box_in = col0 + cbase < p.N;
                if (tile_rows_ok) {
                    if (!box_in)
                        continue;
                    const uint32_t stg = smem_addr(epi_stage + (bx % Cfg::EPI_BUFS) * Cfg::EPI_BOX_BYTES);
                    if (threadIdx.x == 0)
                        bulk_wait_group_read<Cfg::EPI_BUFS - 1>();
                    named_barrier_sync(1, 128);
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        if (ch * 8 < ncols) {
                            const uint32_t off =
                                full ? static_cast<uint32_t>(row * 128 + ((ch ^ (row & 7)) * 16))
                                     : static_cast<uint32_t>(row * ncols * 2 + ch * 16);
                            st_shared_v4(stg + off, pack_bf16x8(v + ch * 8));
                        }
                    }
                    fence_proxy_async_smem();
                    named_barrier_sync(1, 128);
                    if (threadIdx.x == 0) {
                        tma_store_2d(full ? static_cast<const void *>(&tmap_d64)
                                          : static_cast<const void *>(&tmap_drem),
                                     stg, col0 + cbase, grow0);
                        bulk_commit_group();
                    }
                } else if (row_ok && box_in) {
                    const size_t grow = static_cast<size_t>(grow0) + row;
                    __nv_bfloat16 *drow = p.D + grow * p.N + col0 + cbase;
#pragma unroll
                    for (int c = 0; c < 64; c += 8)
                        if (c < ncols && col0 + cbase + c < p.N)
                            *reinterpret_cast<uint4 *>(drow + c) = pack_bf16x8(v + c);
                }
            }
            ++acc_i;
        }
        if (threadIdx.x == 0)
            bulk_wait_group<0>();
        __syncwarp();
    }

    __syncthreads();
    // no CTA leaves (or frees TMEM) while its peer may still signal its
    // barriers or the leader's MMAs may still write its TMEM
    cluster_sync();
    if (warp == Cfg::MMA_WARP) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
    }
}

// ---------------------------------------------- scale packing (boundary)
//
// fp32 scales -> packed UE8M0 words, four K blocks per int32, byte j of
// word (b, g, r) = K block 4g + j (127, i.e. scale 1, past the last block
// and for pad rows).  A float32 power of two 2^(E-127) with a zero mantissa
// has the UE8M0 code E (the two formats share the bias); 2^-127 is the
// float32 subnormal 0x00400000 and has code 0.  Anything else is not a
// UE8M0 value: its byte becomes 255 (NaN) and kCodeBadScale is recorded.
//   mn_major: sf [batch][nkb][out_ld] (out_ld = rows rounded up to 4)
//   else    : sf [batch][rows][nkb]   (out_ld = rows)
//   out     : [batch][ceil(nkb/4)][out_ld]
__global__ void transform_sf_ue8m0_kernel(const float *__restrict__ sf, int32_t *__restrict__ out, int rows,
                                          int out_ld, int nkb, int batch, int mn_major)
{
    const int ngroups = (nkb + 3) / 4;
    const int64_t total = static_cast<int64_t>(batch) * ngroups * out_ld;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int r = static_cast<int>(idx % out_ld);
        const int64_t bg = idx / out_ld;
        const int g = static_cast<int>(bg % ngroups);
        const int64_t b = bg / ngroups;
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int kb = 4 * g + j;
            uint32_t code = 127;
            if (r < rows && kb < nkb) {
                const float v = mn_major ? sf[(b * nkb + kb) * out_ld + r] : sf[(b * rows + r) * nkb + kb];
                const uint32_t bits = __float_as_uint(v);
                const uint32_t e = bits >> 23;  // sign bit included: must be 0
                if ((bits & 0x7FFFFFu) == 0 && e >= 1 && e <= 254) {
                    code = e;
                } else if (bits == 0x00400000u) {
                    code = 0;
                } else {
                    code = 255;
                    record_status(kCodeBadScale, kRoleTransform, 0);
                }
            }
            word |= code << (8 * j);
        }
        out[idx] = static_cast<int32_t>(word);
    }
}

}  // namespace dg
