// fp8_gemm_bs_kernel.cuh -- the UE8M0 block-scaled mode of the FP8 GEMM on
// sm_100a (dense, contiguous-grouped and masked-grouped layouts), on one-CTA
// 128 x BN tiles or on 256 x BN tiles shared by the two CTAs of a cluster.
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
// B200 design of one CTA (one per SM, persistent over tiles):
//   warp 4 (A producer) : per stage of KS K blocks, one 3-D TMA box of A
//                         (its own 128 rows);
//   warp 5 (B producer) : the same for B (BN rows, or BN/2 on a pair); each
//                         TMA instruction costs its issuing warp a roughly
//                         fixed time, so A and B go through different warps;
//   warp 6 (scale loader): copies the packed scale words of the tile's rows
//                         of A and B, one K-block group (four K blocks) at a
//                         time, into a 4-slot staging ring in shared memory
//                         (cp.async, each lane's copies arriving on the
//                         slot's barrier as they land);
//   warps 8-11 (scale writers): per group, warp q reads the staged words of
//                         its lane and writes them with tcgen05.st into its
//                         32-lane quarter of a TMEM scale slot (32 rows x 4
//                         columns per 128 rows: TMEM lane r, column j holds
//                         the scale of row r + 32 j, the same in all four
//                         quarters), then announces the slot;
//   warp 7 (MMA)        : (the pair's rank-0 CTA) 4 block-scaled MMAs per K
//                         block into one of two TMEM accumulators, reading
//                         the group's scale slot; commits free the stage, the
//                         scale slot and hand over the finished tile;
//   warps 0-3 (epilogue): read the finished accumulator from TMEM (thread t =
//                         tile row t), free it, round to bf16 and TMA-store
//                         64-column boxes (row by row where a grouped layout
//                         must leave rows untouched).
// On a pair (cta_group::2) each CTA loads its own 128 rows of A and half of
// B's rows, both CTAs' boxes signal the leader's full barrier, each CTA's
// scale writers fill its own TMEM with the scales of its 128 rows of A and
// of all BN rows of B and arrive on the leader's barrier, and the leader's
// commits arrive on both CTAs' barriers (multicast arrive, not a data copy).
// Per SM and K block the operand bytes then drop from (128 + BN) * 128 to
// (128 + BN/2) * 128.
// Dense problems with too few tiles to fill the GPU (decode shapes) split
// each tile's K range over a cluster of CTAs instead: each writes its fp32
// partial tile to an L2-resident workspace, and after a cluster barrier each
// sums a slice of the tile's rows over the partials in a fixed order.
//
// Waits are bounded: a wait that runs out records DG_ERR_TIMEOUT, raises the
// CTA's (and on a pair its peer's) abort flag and every role leaves; copies
// and MMAs in flight are drained and TMEM freed before exit.
#pragma once

#include <type_traits>

#include "fp8_gemm_kernel.cuh"
#include "fp8_gemm_pair_kernel.cuh"

namespace dg {

// The scale loader's copy of one K-block group (four K blocks): lane r
// copies the packed words of rows r, r+32, r+64, r+96 of the tile's 128 rows
// of A and of each 128-row chunk of its BN rows of B into a staging slot
// (16 bytes per row of a chunk), with cp.async, and each lane's copies
// arrive on the slot's barrier when they land (so the loader never waits for
// them).  Rows past the matrix are zero-filled (their operand rows are zero
// too).
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

// BN: tile width; STAGES: ring depth; KS: 128-wide K blocks per stage; PAIR:
// 256-row tiles on a CTA pair; SPLIT: (dense, one-CTA) the K range of each
// tile split over the CTAs of a cluster, whose fp32 partial tiles meet in an
// L2-resident workspace and are summed in a fixed order.
template <int BN_, int STAGES_, int KS_, bool PAIR_, bool SPLIT_ = false>
struct BsConfig {
    static constexpr int BN = BN_;
    static constexpr int STAGES = STAGES_;
    static constexpr int KS = KS_;
    static constexpr bool PAIR = PAIR_;
    static constexpr bool SPLIT = SPLIT_;
    static constexpr int B_ROWS = PAIR ? BN / 2 : BN;  // rows of B this CTA loads
    static constexpr int NUM_EPI_WARPS = 4;
    static constexpr int PRODUCER_A = 4;
    static constexpr int PRODUCER_B = 5;
    static constexpr int SF_LOADER = 6;
    static constexpr int MMA_WARP = 7;
    static constexpr int SF_WRITER0 = 8;  // warps 8-11, one per TMEM lane quarter
    static constexpr int THREADS = 12 * 32;
    static constexpr int A_BYTES = kBM * kBK;
    static constexpr int B_BYTES = B_ROWS * kBK;
    static constexpr int STAGE_A = KS * A_BYTES;
    static constexpr int STAGE_B = KS * B_BYTES;
    static constexpr int SFB_CHUNKS = (BN + 127) / 128;
    static constexpr int SF_GROUP_BYTES = 512 * (1 + SFB_CHUNKS);  // one group's staged words
    static constexpr int SF_RING = 4;                              // staging slots
    // TMEM: two fp32 accumulators, then scale slots of 16 columns (A: 4,
    // B: 4 per 128 columns), as many as fit up to 4.
    static constexpr int ACC_STRIDE = (BN + 31) / 32 * 32;
    static constexpr int NACC = 2;
    static constexpr int SF_COL0 = NACC * ACC_STRIDE;
    static constexpr int SF_SLOT_COLS = 16;
    static constexpr int TSLOTS = (512 - SF_COL0) / SF_SLOT_COLS >= 4 ? 4 : (512 - SF_COL0) / SF_SLOT_COLS;
    static constexpr int TMEM_COLS = SF_COL0 + TSLOTS * SF_SLOT_COLS <= 256 ? 256 : 512;
    // (+ one barrier for the K-split reduction's TMA load)
    static constexpr int BAR_BYTES = 8 * (2 * STAGES + 2 * NACC + 2 * SF_RING + 2 * TSLOTS + 1) + 16;
    // K split: the reduction reads this CTA's rows of all S partials
    // (BN/4 x 128 float4s whatever S is) into the idle operand ring at
    // offset 0, and stages its bf16 rows (at most 64 x BN) after them.
    static constexpr int RED_IN_BYTES = (BN / 4) * kBM * 16;
    static constexpr int RED_OUT_OFFSET = (RED_IN_BYTES + 1023) / 1024 * 1024;
    static constexpr int EPI_FULL_BOXES = BN / 64;
    static constexpr int EPI_REM = BN % 64;
    static constexpr int EPI_BOXES = EPI_FULL_BOXES + (EPI_REM > 0 ? 1 : 0);
    static constexpr int EPI_BOX_BYTES = kBM * 128;
    static constexpr int PIPE_BYTES = STAGES * (STAGE_A + STAGE_B) + SF_RING * SF_GROUP_BYTES;
    static constexpr int EPI_OFFSET = (PIPE_BYTES + BAR_BYTES + 1023) / 1024 * 1024;
    static constexpr int EPI_BUFS = 1024 + EPI_OFFSET + 2 * EPI_BOX_BYTES <= 232448 ? 2 : 1;
    // (a split kernel writes its partial tile to global memory: no staging)
    static constexpr int SMEM_BYTES = 1024 + EPI_OFFSET + (SPLIT ? 0 : EPI_BUFS * EPI_BOX_BYTES);

    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N: multiple of 16, <= 256");
    static_assert(!PAIR || BN % 32 == 0, "a pair tile's B half must be whole 16-row TMA boxes");
    static_assert(EPI_REM % 8 == 0, "remainder box must be whole 16-byte chunks");
    static_assert(KS == 1 || KS == 2 || KS == 4, "K blocks per stage");
    static_assert(!SPLIT || (!PAIR && BN % 4 == 0), "K split: one-CTA tiles, float4 partial columns");
    static_assert(SF_COL0 % 16 == 0 && TSLOTS >= 2, "accumulators and two scale slots must fit in TMEM");
    static_assert(4 + 4 * SFB_CHUNKS <= SF_SLOT_COLS, "scale slot too small");
    static_assert(B_BYTES % 1024 == 0, "B tiles must keep 1024-byte swizzle atoms aligned");
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
    static_assert(!SPLIT || RED_OUT_OFFSET + 64 * BN * 2 <= STAGES * (STAGE_A + STAGE_B),
                  "the split reduction's buffers fit in the operand ring");
};

template <int BN, int STAGES, int KS, int LAYOUT, bool PAIR, bool SPLIT = false>
__global__ void __launch_bounds__(BsConfig<BN, STAGES, KS, PAIR, SPLIT>::THREADS, 1)
    fp8_gemm_bs_kernel(const __grid_constant__ CUtensorMap tmap_a,
                       const __grid_constant__ CUtensorMap tmap_b,
                       const __grid_constant__ CUtensorMap tmap_d64,
                       const __grid_constant__ CUtensorMap tmap_drem, const GemmParams p)
{
    using Cfg = BsConfig<BN, STAGES, KS, PAIR, SPLIT>;
    using Sched = std::conditional_t<PAIR, PairScheduler<LAYOUT>, TileScheduler<LAYOUT, SPLIT>>;
    static_assert(LAYOUT == kDense || LAYOUT == kContiguous || LAYOUT == kMasked,
                  "block-scaled mode: dense, contiguous and masked layouts");
    static_assert(!SPLIT || LAYOUT == kDense, "the K split is implemented for the dense layout");
    constexpr int NACC = Cfg::NACC;
    constexpr int TSLOTS = Cfg::TSLOTS;
    constexpr int TILE_ROWS = PAIR ? kPairBM : kBM;
    constexpr uint32_t CTAS = PAIR ? 2 : 1;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *a_tiles = smem;                              // [STAGES][KS][128][128 B]
    uint8_t *b_tiles = smem + STAGES * Cfg::STAGE_A;      // [STAGES][KS][B_ROWS][128 B]
    uint8_t *sf_ring = b_tiles + STAGES * Cfg::STAGE_B;   // [SF_RING][1+SFB_CHUNKS][32][16 B]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sf_ring + Cfg::SF_RING * Cfg::SF_GROUP_BYTES);
    uint64_t *full_bar = bars;                     // (leader) A and B boxes of the stage landed
    uint64_t *empty_bar = bars + STAGES;           // MMAs of the stage done
    uint64_t *tfull_bar = bars + 2 * STAGES;       // accumulator holds a finished tile
    uint64_t *tempty_bar = tfull_bar + NACC;       // (leader) accumulator read out by every CTA
    uint64_t *staged_full = tempty_bar + NACC;     // staging slot holds its group's words
    uint64_t *staged_empty = staged_full + Cfg::SF_RING;  // scale writers are done with the slot
    uint64_t *sf_full = staged_empty + Cfg::SF_RING;      // (leader) TMEM scale slot written by every CTA
    uint64_t *sf_empty = sf_full + TSLOTS;                // MMAs reading the scale slot done
    uint64_t *red_bar = sf_empty + TSLOTS;                 // K split: the reduction's partials landed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(red_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    uint8_t *epi_stage = smem + Cfg::EPI_OFFSET;

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    stamp_start(p);

    if (warp == Cfg::PRODUCER_A && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_addr(full_bar + s), 2);  // the (leader's) A and B expect-tx arrivals
            mbar_init(smem_addr(empty_bar + s), 1);
        }
        for (int b = 0; b < NACC; ++b) {
            mbar_init(smem_addr(tfull_bar + b), 1);
            mbar_init(smem_addr(tempty_bar + b), CTAS * Cfg::NUM_EPI_WARPS);
        }
        for (int r = 0; r < Cfg::SF_RING; ++r) {
            mbar_init(smem_addr(staged_full + r), 32);  // one cp.async arrival per loader lane
            mbar_init(smem_addr(staged_empty + r), 4);  // the four scale writers
        }
        for (int t = 0; t < TSLOTS; ++t) {
            mbar_init(smem_addr(sf_full + t), CTAS * 4);
            mbar_init(smem_addr(sf_empty + t), 1);
        }
        mbar_init(smem_addr(red_bar), 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmap_a);
        tma_prefetch_desc(&tmap_b);
        // (K split: tmap_d64 describes the partials, tmap_drem the
        // reduction's output rows)
        if (SPLIT || Cfg::EPI_FULL_BOXES > 0)
            tma_prefetch_desc(&tmap_d64);
        if (SPLIT || Cfg::EPI_REM > 0)
            tma_prefetch_desc(&tmap_drem);
    }
    if (warp == Cfg::MMA_WARP) {
        if constexpr (PAIR) {
            tmem_alloc_pair(smem_addr(tmem_slot), Cfg::TMEM_COLS);
            tmem_relinquish_alloc_permit_pair();
        } else {
            tmem_alloc(smem_addr(tmem_slot), Cfg::TMEM_COLS);
            tmem_relinquish_alloc_permit();
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if constexpr (PAIR)
        cluster_sync();  // both CTAs' barriers exist before either signals the other
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    const uint64_t tmo = p.timeout_ns;
    const uint64_t drain_tmo = tmo > 1000000000ull ? tmo : 1000000000ull;
    const uint32_t peer_abort =
        PAIR ? map_shared_rank(smem_addr(const_cast<int *>(abort_flag)), rank ^ 1u) : 0u;
    // the leader's barriers as seen from this CTA
    const uint32_t full_lead = PAIR ? map_shared_rank(smem_addr(full_bar), 0) : smem_addr(full_bar);
    const uint32_t tempty_lead = PAIR ? map_shared_rank(smem_addr(tempty_bar), 0) : smem_addr(tempty_bar);
    const uint32_t sf_full_lead = PAIR ? map_shared_rank(smem_addr(sf_full), 0) : smem_addr(sf_full);
    // a bounded wait of the whole warp (a pair CTA that gives up also stops
    // its peer)
    auto wait = [&](uint32_t bar, uint32_t parity, uint32_t role, uint32_t tag) {
        if constexpr (PAIR)
            return pair_warp_wait(bar, parity, tmo, abort_flag, peer_abort, role, tag);
        else
            return warp_wait_bounded(bar, parity, tmo, abort_flag, role, tag);
    };
    // arrive on a barrier of the leader CTA (local on a one-CTA tile)
    auto arrive_lead = [&](uint32_t bar_lead) {
        if constexpr (PAIR)
            mbar_arrive_cluster(bar_lead);
        else
            mbar_arrive(bar_lead);
    };
    // this CTA's K blocks [kb_lo, kb_hi) of the current tile (a K split gives
    // each CTA of the cluster its share; a stage may then straddle two
    // groups of four K blocks, so the scale slots go by K block)
    auto kb_lo = [&](const Sched &sc) {
        if constexpr (SPLIT)
            return sc.kb_begin();
        else
            return 0;
    };
    auto kb_hi = [&](const Sched &sc) {
        if constexpr (SPLIT)
            return sc.kb_end();
        else
            return p.num_kb;
    };

    if (warp == Cfg::PRODUCER_A || warp == Cfg::PRODUCER_B) {
        // ------------------------------------------------- TMA producers
        const bool is_a = warp == Cfg::PRODUCER_A;
        Sched sched(p);
        TileCoord tc;
        uint32_t stage = 0, phase = 0, issued = 0;
        bool ok = !(p.stall_injection && blockIdx.x < CTAS && blockIdx.y == 0 && blockIdx.z == 0);
        while (ok && sched.next(tc, is_a && leader && lane == 0)) {
            const int row = is_a ? (LAYOUT == kMasked ? tc.g * p.M : 0) + tc.mb * TILE_ROWS +
                                       static_cast<int>(rank) * kBM
                                 : tc.g * p.N + tc.nb * BN + static_cast<int>(rank) * Cfg::B_ROWS;
            for (int kb0 = kb_lo(sched); kb0 < kb_hi(sched); kb0 += KS) {
                if (!wait(smem_addr(empty_bar + stage), phase ^ 1, kRoleProducer, stage)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = full_lead + 8 * stage;
                if (elect_one()) {
                    const int bytes = is_a ? Cfg::STAGE_A : Cfg::STAGE_B;
                    const uint32_t dst = is_a ? smem_addr(a_tiles + stage * Cfg::STAGE_A)
                                              : smem_addr(b_tiles + stage * Cfg::STAGE_B);
                    const void *map = is_a ? static_cast<const void *>(&tmap_a) : static_cast<const void *>(&tmap_b);
                    if constexpr (PAIR) {
                        if (leader)
                            mbar_arrive_expect_tx(smem_addr(full_bar + stage), 2 * bytes);
                        // dense: A rows are read again by the band's other
                        // column tiles while B streams past -- keep them in
                        // L2 (measured: prefill 489 -> 456 us; on the
                        // contiguous layout, whose K range is short, it cost
                        // 2%, so only the dense layout takes the hint)
                        if (LAYOUT == kDense && is_a)
                            tma_load_3d_pair_hint(dst, map, fb, 0, row, kb0, l2_policy_evict_last());
                        else
                            tma_load_3d_pair(dst, map, fb, 0, row, kb0);
                    } else {
                        mbar_arrive_expect_tx(fb, bytes);
                        tma_load_3d(dst, map, fb, 0, row, kb0);
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
        if constexpr (PAIR) {
            // On the normal path every box has landed (the leader's MMA waited
            // for it).  After an abort, boxes may still be in flight towards a
            // barrier or tile of either CTA: give them a bounded moment to land
            // before the pair passes the exit barrier.
            if (!ok && lane == 0) {
                const uint64_t t0 = global_timer_ns();
                while (global_timer_ns() - t0 < 200000ull) {
                }
            }
        } else {
            // the copies of the last min(STAGES, issued) stages land before exit
            if (lane == 0) {
                const uint32_t first = issued > STAGES ? issued - STAGES : 0;
                for (uint32_t i = first; i < issued; ++i)
                    wait_bounded(smem_addr(full_bar + i % STAGES), (i / STAGES) & 1, drain_tmo, abort_flag,
                                 kRoleDrain, i % STAGES, false);
            }
        }
        __syncwarp();
    } else if (warp == Cfg::SF_LOADER) {
        // ------------------------------------------------- scale loader
        // Each K-block group's scale words into the staging ring as soon as a
        // slot is free, up to SF_RING groups ahead of the writers.
        Sched sched(p);
        TileCoord tc;
        uint32_t gs = 0;  // group sequence number over all tiles
        bool ok = true;
        while (ok && sched.next(tc, false)) {
            const int32_t *sfa_g =
                p.sfa + (LAYOUT == kMasked ? static_cast<size_t>(tc.g) * p.num_kg * p.sfa_ld : 0);
            const int32_t *sfb_g = p.sfb + static_cast<size_t>(tc.g) * p.num_kg * p.nbn;
            const int a_row0 = tc.mb * TILE_ROWS + static_cast<int>(rank) * kBM + lane;
            const int n_row0 = tc.nb * BN + lane;
            const int kg_hi = (kb_hi(sched) - 1) / 4;
            for (int kg = kb_lo(sched) / 4; kg <= kg_hi; ++kg, ++gs) {
                const uint32_t slot = gs % Cfg::SF_RING, sph = (gs / Cfg::SF_RING) & 1;
                if (!wait(smem_addr(staged_empty + slot), sph ^ 1, kRoleProducer, 96 + slot)) {
                    ok = false;
                    break;
                }
                sf_load_group<Cfg::SFB_CHUNKS>(smem_addr(sf_ring + slot * Cfg::SF_GROUP_BYTES),
                                               smem_addr(staged_full + slot), sfa_g, sfb_g, p, a_row0, n_row0, kg);
            }
        }
        cp_async_wait_all();  // no copy still in flight at exit
    } else if (warp >= Cfg::SF_WRITER0) {
        // ------------------------------------------------- scale writers
        // Warp q writes TMEM lanes 32q..32q+31 of the group's scale slot: 4
        // columns for A (lane r, column j = the scale word of row r + 32j)
        // and 4 per 128 columns of B, the same words in every quarter.
        const uint32_t lane_bits = static_cast<uint32_t>((warp % 4) * 32) << 16;
        Sched sched(p);
        TileCoord tc;
        uint32_t gs = 0;
        bool ok = true;
        while (ok && sched.next(tc, false)) {
            const int kg_hi = (kb_hi(sched) - 1) / 4;
            for (int kg = kb_lo(sched) / 4; kg <= kg_hi; ++kg, ++gs) {
                const uint32_t rslot = gs % Cfg::SF_RING, rph = (gs / Cfg::SF_RING) & 1;
                const uint32_t tslot = gs % TSLOTS, tph = (gs / TSLOTS) & 1;
                if (!wait(smem_addr(staged_full + rslot), rph, kRoleProducer, 112 + rslot) ||
                    !wait(smem_addr(sf_empty + tslot), tph ^ 1, kRoleProducer, 120 + tslot)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t src = smem_addr(sf_ring + rslot * Cfg::SF_GROUP_BYTES) + 16 * lane;
                uint4 w[1 + Cfg::SFB_CHUNKS];
#pragma unroll
                for (int c = 0; c < 1 + Cfg::SFB_CHUNKS; ++c)
                    w[c] = ld_shared_v4u(src + 512 * c);
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(smem_addr(staged_empty + rslot));
                const uint32_t taddr = tmem_base + lane_bits + Cfg::SF_COL0 + tslot * Cfg::SF_SLOT_COLS;
#pragma unroll
                for (int c = 0; c < 1 + Cfg::SFB_CHUNKS; ++c)
                    tmem_st_32x32b_x4(taddr + 4 * c, w[c]);
                tmem_st_wait();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0)
                    arrive_lead(sf_full_lead + 8 * tslot);
            }
        }
    } else if (warp == Cfg::MMA_WARP) {
        // ------------------------------------------------ MMA issuer (leader)
        if (leader) {
            Sched sched(p);
            TileCoord tc;
            uint32_t stage = 0, phase = 0, acc_i = 0, gs = 0;
            uint32_t last_bar = 0, last_parity = 0;
            bool ok = true;
            const uint64_t a_desc0 = smem_desc_k_sw128(smem_addr(a_tiles));
            const uint64_t b_desc0 = smem_desc_k_sw128(smem_addr(b_tiles));
            while (ok && sched.next(tc, false)) {
                const uint32_t buf = acc_i % NACC, tph = (acc_i / NACC) & 1;
                if (!wait(smem_addr(tempty_bar + buf), tph ^ 1, kRoleMma, 16 + buf)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + buf * Cfg::ACC_STRIDE;
                const int kbl = kb_lo(sched), kbh = kb_hi(sched);
                for (int kb0 = kbl; kb0 < kbh; kb0 += KS) {
                    if (!wait(smem_addr(full_bar + stage), phase, kRoleMma, stage)) {
                        ok = false;
                        break;
                    }
#pragma unroll
                    for (int q = 0; q < KS; ++q) {
                        const int kb = kb0 + q;
                        if (kb >= kbh)
                            break;
                        // the K block's scale slot: its group's sequence number
                        const uint32_t g = gs + static_cast<uint32_t>(kb / 4 - kbl / 4);
                        const uint32_t tslot = g % TSLOTS;
                        if ((kb == kbl || kb % 4 == 0) &&
                            !wait(smem_addr(sf_full + tslot), (g / TSLOTS) & 1, kRoleMma, 24 + tslot)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        const uint32_t sf_col = tmem_base + Cfg::SF_COL0 + tslot * Cfg::SF_SLOT_COLS;
                        const bool group_done = kb + 1 == kbh || (kb + 1) % 4 == 0;
                        if (elect_one()) {
                            const uint32_t byte = static_cast<uint32_t>(kb & 3);
                            const uint32_t idesc = idesc_mxf8_e4m3_ue8m0(TILE_ROWS, BN, byte);
                            const uint64_t ad =
                                a_desc0 + static_cast<uint64_t>((stage * Cfg::STAGE_A + q * Cfg::A_BYTES) >> 4);
                            const uint64_t bd =
                                b_desc0 + static_cast<uint64_t>((stage * Cfg::STAGE_B + q * Cfg::B_BYTES) >> 4);
#pragma unroll
                            for (int j = 0; j < kBK / 32; ++j) {
                                const uint32_t acc = (kb > kbl || j > 0) ? 1u : 0u;
                                if constexpr (PAIR)
                                    mma_mxf8f6f4_bs_pair(d_tmem, ad + 2 * j, bd + 2 * j, idesc, sf_col | (byte << 30),
                                                         (sf_col + 4) | (byte << 30), acc);
                                else
                                    mma_mxf8f6f4_bs(d_tmem, ad + 2 * j, bd + 2 * j, idesc, sf_col | (byte << 30),
                                                    (sf_col + 4) | (byte << 30), acc);
                            }
                            if (group_done) {
                                if constexpr (PAIR)
                                    mma_commit_pair_multicast(smem_addr(sf_empty + tslot), 0x3);
                                else
                                    mma_commit(smem_addr(sf_empty + tslot));
                            }
                        }
                        __syncwarp();
                    }
                    if (!ok)
                        break;
                    if (elect_one()) {
                        if constexpr (PAIR)
                            mma_commit_pair_multicast(smem_addr(empty_bar + stage), 0x3);
                        else
                            mma_commit(smem_addr(empty_bar + stage));
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
                gs += static_cast<uint32_t>((kbh - 1) / 4 - kbl / 4 + 1);
                if (elect_one()) {
                    if constexpr (PAIR)
                        mma_commit_pair_multicast(smem_addr(tfull_bar + buf), 0x3);
                    else
                        mma_commit(smem_addr(tfull_bar + buf));
                }
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
        const int quad = warp;             // TMEM lane quarter of this warp
        const int row = quad * 32 + lane;  // row within this CTA's 128 == TMEM lane
        const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
        Sched sched(p);
        TileCoord tc;
        uint32_t acc_i = 0;
        bool ok = true;
        while (ok && sched.next(tc, false)) {
            const uint32_t buf = acc_i % NACC, tph = (acc_i / NACC) & 1;
            ok = wait(smem_addr(tfull_bar + buf), tph, kRolePromote, 16 + buf);
            // a warp that gave up takes the others with it (no warp may be
            // left waiting at a later named barrier)
            if (!named_barrier_and(1, 128, ok)) {
                if constexpr (SPLIT) {
                    // this split has no partial: NaN in its workspace slot,
                    // so the cluster's sums show the failure instead of
                    // adding a stale partial left there by an earlier call
                    const size_t tile = static_cast<size_t>(tc.mb) * p.num_nb + tc.nb;
                    float4 *dst = reinterpret_cast<float4 *>(p.ws) +
                                  (tile * p.ksplit + cluster_ctarank()) * (BN / 4) * kBM + row;
                    const float nan = __int_as_float(0x7FC00000);
                    for (int c4 = 0; c4 < BN / 4; ++c4)
                        dst[c4 * kBM] = make_float4(nan, nan, nan, nan);
                }
                ok = false;
                break;
            }
            tc_fence_after_sync();
            const int m_half = tc.mb * TILE_ROWS + static_cast<int>(rank) * kBM;  // this CTA's first row
            const int m_local = m_half + row;
            bool row_ok;
            if constexpr (LAYOUT == kDense) {
                row_ok = m_local < p.M;
            } else if constexpr (LAYOUT == kContiguous) {
                row_ok = false;
                // computed when the row's index is this visit's group and
                // the group of its own 128-row block (its first row's)
                const int block_g = m_half < p.M ? __ldg(p.m_indices + m_half) : -1;
                if (m_local < p.M && block_g >= 0) {
                    const int idx = __ldg(p.m_indices + m_local);
                    row_ok = idx == tc.g && idx == block_g;
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
                float v[64];
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    v[i] = __uint_as_float(r[i]);
                if (bx == Cfg::EPI_BOXES - 1) {
                    // the whole accumulator is in registers: hand it back
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0)
                        arrive_lead(tempty_lead + 8 * buf);
                }
                if constexpr (SPLIT) {
                    // this split's fp32 partial of the box to the workspace,
                    // [tile][split][BN/4][128][4]: a warp's 32 rows write 512
                    // contiguous bytes per column quad
                    const size_t tile = static_cast<size_t>(tc.mb) * p.num_nb + tc.nb;
                    float4 *dst = reinterpret_cast<float4 *>(p.ws) +
                                  ((tile * p.ksplit + cluster_ctarank()) * (BN / 4) + cbase / 4) * kBM + row;
#pragma unroll
                    for (int c = 0; c < 64; c += 4)
                        if (c < ncols)
                            dst[(c / 4) * kBM] = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
                    continue;
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
        if constexpr (SPLIT)
            __threadfence();  // the partial tile is visible to the cluster's reduction
        __syncwarp();
    }

    __syncthreads();
    if constexpr (PAIR) {
        // no CTA leaves (or frees TMEM) while its peer may still signal its
        // barriers or the leader's MMAs may still write its TMEM
        cluster_sync();
    }
    if constexpr (SPLIT) {
        cluster_sync();  // every split's partial tile is in the workspace
        // CTA `rank` sums rows [rank*128/S, (rank+1)*128/S) of the tile over
        // the S partials in split order (a fixed order: results do not
        // depend on timing) and rounds them to bf16.
        const int S = p.ksplit;
        const uint32_t rank_s = cluster_ctarank();
        Sched sched(p);
        TileCoord tc;
        if (sched.next(tc, false)) {
            const int rows_per = kBM / S;
            constexpr int C4 = BN / 4;
            const size_t tile = static_cast<size_t>(tc.mb) * p.num_nb + tc.nb;
            const float4 *src0 = reinterpret_cast<const float4 *>(p.ws) + tile * S * C4 * kBM;
            if (S >= 2 && kBM % S == 0) {
                // (the same condition under which the host built the two maps)
                // One TMA box brings this CTA's rows of all S partials,
                // [S][C4][rows_per] float4s, into the idle operand ring; the
                // sums (in split order) are rounded, staged as
                // [rows_per][BN] bf16 and stored with one TMA box (rows past
                // M and columns past N are clipped).
                const float4 *red_in = reinterpret_cast<const float4 *>(smem);
                uint8_t *red_out = smem + Cfg::RED_OUT_OFFSET;
                const int r0 = static_cast<int>(rank_s) * rows_per;
                if (threadIdx.x == 0) {
                    // the partials were written by generic-proxy stores
                    fence_proxy_async_global();
                    mbar_arrive_expect_tx(smem_addr(red_bar), Cfg::RED_IN_BYTES);
                    tma_load_4d(smem_addr(smem), &tmap_d64, smem_addr(red_bar), 4 * r0, 0, 0,
                                static_cast<int>(tile));
                }
                // the box must land whatever the abort flag says: this CTA's
                // shared memory may not be left while the copy is in flight
                int got_lane = 0;
                if (lane == 0)
                    got_lane = wait_bounded(smem_addr(red_bar), 0, drain_tmo, abort_flag, kRoleDrain, 40, false)
                                   ? 1 : 0;
                const bool got = __shfl_sync(0xFFFFFFFFu, got_lane, 0) != 0;
                if (got) {
                    for (int it = threadIdx.x; it < rows_per * C4; it += Cfg::THREADS) {
                        const int lr = it % rows_per;  // rows fastest: conflict-free reads
                        const int c4 = it / rows_per;
                        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
                        for (int src = 0; src < S; ++src) {
                            const float4 v = red_in[(src * C4 + c4) * rows_per + lr];
                            sum.x += v.x;
                            sum.y += v.y;
                            sum.z += v.z;
                            sum.w += v.w;
                        }
                        __nv_bfloat162 h0 = __floats2bfloat162_rn(sum.x, sum.y);
                        __nv_bfloat162 h1 = __floats2bfloat162_rn(sum.z, sum.w);
                        uint2 u;
                        u.x = *reinterpret_cast<uint32_t *>(&h0);
                        u.y = *reinterpret_cast<uint32_t *>(&h1);
                        *reinterpret_cast<uint2 *>(red_out + (lr * BN + 4 * c4) * 2) = u;
                    }
                }
                fence_proxy_async_smem();
                if (__syncthreads_and(got ? 1 : 0) && threadIdx.x == 0) {
                    tma_store_2d(&tmap_drem, smem_addr(red_out), tc.nb * BN, tc.mb * kBM + r0);
                    bulk_commit_group();
                    bulk_wait_group<0>();
                }
            } else
            for (int it = threadIdx.x; it < rows_per * C4; it += Cfg::THREADS) {
                const int lr = it % rows_per;  // rows fastest: contiguous reads
                const int c4 = it / rows_per;
                const int r = static_cast<int>(rank_s) * rows_per + lr;
                // all S loads in flight at once (S <= 16), then the sum in
                // split order
                float4 w[16];
#pragma unroll
                for (int src = 0; src < 16; ++src)
                    if (src < S)
                        w[src] = __ldcg(src0 + (static_cast<size_t>(src) * C4 + c4) * kBM + r);
                float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int src = 0; src < 16; ++src) {
                    if (src < S) {
                        sum.x += w[src].x;
                        sum.y += w[src].y;
                        sum.z += w[src].z;
                        sum.w += w[src].w;
                    }
                }
                const int grow = tc.mb * kBM + r;
                const int gcol = tc.nb * BN + c4 * 4;
                if (grow < p.M && gcol < p.N) {
                    __nv_bfloat162 h0 = __floats2bfloat162_rn(sum.x, sum.y);
                    __nv_bfloat162 h1 = __floats2bfloat162_rn(sum.z, sum.w);
                    uint2 u;
                    u.x = *reinterpret_cast<uint32_t *>(&h0);
                    u.y = *reinterpret_cast<uint32_t *>(&h1);
                    *reinterpret_cast<uint2 *>(p.D + static_cast<size_t>(grow) * p.N + gcol) = u;
                }
            }
        }
    }
    stamp_end(p);
    if (warp == Cfg::MMA_WARP) {
        tc_fence_after_sync();
        if constexpr (PAIR)
            tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
        else
            tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
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
