// fp8_gemm_pair_kernel.cuh -- the fine-grained-scaled FP8 GEMM on CTA pairs
// (2-SM tcgen05 MMA, cta_group::2) for problems with enough 256-row tiles to
// fill the GPU.
//
// Same method as fp8_gemm_kernel.cuh (DeepGEMM pages: per-128-K partials on
// the tensor cores, promoted on the CUDA cores as
// acc += sA[m,kb] * sB[n/128,kb] * partial; lqnn.cn article, section
// "DeepGEMM"), on a 256 x BN tile shared by the two CTAs of a cluster, one
// per SM:
//   * each CTA holds its own 128 rows of A and BN/2 rows of B per K block, so
//     per SM the operand bytes per K block drop from (128 + BN) * 128 to
//     (128 + BN/2) * 128 -- the tensor core of each SM reads the other half
//     of B from the peer's shared memory.  With BN = 256 that is 32 KB per
//     SM per K block instead of 48 KB, which keeps the L2 -> SM feed below
//     the rate at which TMA delivers it;
//   * two producer warps per CTA (one for A, one for B) issue 3-D TMA boxes
//     of KS K blocks each: the engine costs a roughly fixed time per
//     instruction and per issuing warp, so fewer, larger instructions from
//     two warps keep up with the MMA;
//   * both CTAs' boxes signal the full barrier of CTA rank 0 (the leader;
//     cta_group::2 loads, no multicast), whose producers post the expected
//     byte count of both CTAs;
//   * the leader's MMA warp issues tcgen05.mma.cta_group::2 (M = 256); each
//     CTA's TMEM receives its 128 rows.  Its commits arrive on the barriers
//     of both CTAs (tcgen05.commit multicast: an arrive, not a data copy);
//   * each CTA's promotion warps load their partial from TMEM, hand the
//     buffer back to the leader's barrier, and promote with the scales of
//     their own rows, which their own producer copied (cp.async);
//   * each CTA rounds and stores its 128 rows (TMA store, 32-column boxes).
// Every wait is bounded; a CTA that gives up also raises its peer's abort
// flag, and both leave together through the final cluster barrier.
#pragma once

#include "fp8_gemm_kernel.cuh"

namespace dg {

constexpr int kPairBM = 2 * kBM;  // rows of a pair tile

// Tiles of 256 rows for a CTA pair.  Both CTAs run their own copy and see the
// same sequence (blockIdx.x / 2 picks the pair).  The contiguous layout lets
// a pair's two 128-row halves belong to different groups: such a pair row is
// visited twice (once per group) in a second pass over the tile space, and
// each visit stores only the rows of its group.
template <int LAYOUT>
struct PairScheduler {
    const GemmParams &p;
    int next_t, stride;
    int cur_g = 0, cur_base = 0, cur_count = -1;

    __device__ explicit PairScheduler(const GemmParams &params)
        : p(params), next_t(blockIdx.x / 2), stride(gridDim.x / 2) {}

    __device__ bool next(TileCoord &tc, bool report)
    {
        if constexpr (LAYOUT == kMasked) {
            const int t = next_t;
            while (true) {
                if (cur_g >= p.G)
                    return false;
                if (cur_count < 0) {
                    int mm = __ldg(p.masked_m + cur_g);
                    if (mm > p.M || mm < 0) {
                        if (report)
                            record_status(kCodeBadGroup, kRoleSched, cur_g);
                        mm = mm < 0 ? 0 : p.M;
                    }
                    cur_count = ((mm + kPairBM - 1) / kPairBM) * p.num_nb;
                }
                if (t < cur_base + cur_count)
                    break;
                cur_base += cur_count;
                ++cur_g;
                cur_count = -1;
            }
            next_t += stride;
            const int local = t - cur_base;
            const int pms = cur_count / p.num_nb;
            tc.g = cur_g;
            tc.nb = local / pms;
            tc.mb = local - tc.nb * pms;
            return true;
        } else {
            const int total = p.num_mb * p.num_nb;  // num_mb counts 256-row pair rows here
            const int limit = LAYOUT == kContiguous ? 2 * total : total;
            while (next_t < limit) {
                int t = next_t;
                next_t += stride;
                const bool second = t >= total;
                if (second)
                    t -= total;
                const int per = p.raster * p.num_nb;
                const int grp = t / per;
                const int within = t - grp * per;
                const int rows_here = min(p.raster, p.num_mb - grp * p.raster);
                tc.mb = grp * p.raster + within % rows_here;
                tc.nb = within / rows_here;
                tc.g = 0;
                if constexpr (LAYOUT == kContiguous) {
                    const int r0 = tc.mb * kPairBM;
                    const int g0 = __ldg(p.m_indices + r0);
                    const int g1 = r0 + kBM < p.M ? __ldg(p.m_indices + r0 + kBM) : -1;
                    // a half whose first row is out of range, or is padding
                    // over rows that carry a group index, breaks the
                    // alignment rule: its rows stay untouched, and it is
                    // flagged (once, on the first pass, at column block 0)
                    if (report && !second && tc.nb == 0 &&
                        (g0 >= p.G || g1 >= p.G || (g0 < 0 && padding_block_has_rows(p.m_indices, r0)) ||
                         (g1 < 0 && r0 + kBM < p.M && padding_block_has_rows(p.m_indices, r0 + kBM))))
                        record_status(kCodeBadGroup, kRoleSched, 0);
                    const bool v0 = g0 >= 0 && g0 < p.G;
                    const bool v1 = g1 >= 0 && g1 < p.G;
                    if (!second) {
                        if (v0)
                            tc.g = g0;
                        else if (v1)
                            tc.g = g1;
                        else
                            continue;
                    } else {
                        if (v0 && v1 && g1 != g0)
                            tc.g = g1;
                        else
                            continue;
                    }
                }
                return true;
            }
            return false;
        }
    }
};

// NWG promotion warpgroups split the tile's columns (BN / NWG each).  With
// REBAL (always for three or more warpgroups), the block gains an idle
// fourth control warp, so that the two producers, the MMA warp and it form
// one control warpgroup, and registers are rebalanced with setmaxnreg: the
// block is launched at LAUNCH_REGS a thread, the control warpgroup drops to
// CTRL_REGS and the promotion warpgroups take what is left (PROMO_REGS).
// That lets each promotion thread hold its whole partial beside its
// accumulator and load it from TMEM in one round (RMAX = BN_WG), so each
// buffer goes back to the MMA after a single TMEM-load latency.
template <int BN_, int STAGES_, int KS_, int NWG_ = 2, bool REBAL_ = false>
struct PairConfig {
    static constexpr int BN = BN_;          // columns of the pair tile
    static constexpr int BN_HALF = BN / 2;  // B rows held by each CTA
    static constexpr int STAGES = STAGES_;
    static constexpr int KS = KS_;
    static constexpr int NUM_WG = NWG_;     // promotion warpgroups
    static constexpr int BN_WG = BN / NUM_WG;
    static constexpr bool REBALANCE = REBAL_ || NUM_WG >= 3;
    // TMEM load rounds: the whole partial when it fits beside the
    // accumulator, else halves of up to 40 columns, else rounds of 32.
    static constexpr int RMAX =
        (BN_WG <= 64 || (REBALANCE && BN_WG <= 80)) ? BN_WG : (BN_WG <= 80 ? BN_WG / 2 : 32);
    static constexpr int NUM_PROMO_WARPS = 4 * NUM_WG;
    static constexpr int PRODUCER_A_WARP = NUM_PROMO_WARPS;
    static constexpr int PRODUCER_B_WARP = NUM_PROMO_WARPS + 1;
    static constexpr int MMA_WARP = NUM_PROMO_WARPS + 2;
    static constexpr int CTRL_WARPS = REBALANCE ? 4 : 3;
    static constexpr int THREADS = (NUM_PROMO_WARPS + CTRL_WARPS) * 32;
    static constexpr int LAUNCH_REGS = REBALANCE ? (65536 / THREADS) / 8 * 8 : 0;
    static constexpr int CTRL_REGS = 56;
    static constexpr int PROMO_REGS_FIT = REBALANCE ? (LAUNCH_REGS * THREADS - 128 * CTRL_REGS) / (NUM_WG * 128) / 8 * 8 : 0;
    static constexpr int PROMO_REGS = PROMO_REGS_FIT > 256 ? 256 : PROMO_REGS_FIT;
    // Warpgroup columns start at multiples of BN_WG; when BN_WG divides 128
    // they never straddle a 128-wide weight block, so one scale serves them.
    static constexpr bool UNIFORM_SCALE = (128 % (BN / NWG_) == 0) && (BN % (BN / NWG_) == 0);
    static constexpr int A_BYTES = kBM * kBK;      // one K block of this CTA's A rows
    static constexpr int B_BYTES = BN_HALF * kBK;  // one K block of this CTA's B rows
    static constexpr int STAGE_BYTES = KS * (A_BYTES + B_BYTES);
    static constexpr int SA_BYTES = KS * kBM * 4;
    static constexpr int SB_BYTES = KS * 16;
    static constexpr int ACC_STRIDE = (BN + 31) / 32 * 32;
    static constexpr int NBUF = (512 / ACC_STRIDE) < 4 ? (512 / ACC_STRIDE) : 4;
    static constexpr int TMEM_COLS = NBUF * ACC_STRIDE <= 256 ? 256 : 512;
    // full, sfull, empty, sread per stage; tfull, tempty per TMEM buffer
    static constexpr int BAR_BYTES = 8 * (4 * STAGES + 2 * NBUF) + 16;
    // Epilogue boxes of 32 columns (64-byte rows, 64-byte swizzle), one
    // staging buffer per warpgroup, plus one remainder box of the leftover
    // columns (a multiple of 8).
    static constexpr int EPI_BOX = 32;
    static constexpr int EPI_FULL_BOXES = BN_WG / EPI_BOX;
    static constexpr int EPI_REM = BN_WG % EPI_BOX;
    static constexpr int EPI_WG_BYTES = kBM * EPI_BOX * 2;
    static constexpr int PIPE_BYTES = STAGES * (STAGE_BYTES + SA_BYTES + SB_BYTES);
    static constexpr int EPI_OFFSET = (PIPE_BYTES + BAR_BYTES + 1023) / 1024 * 1024;
    // One staging buffer per output box when shared memory allows (as in the
    // one-CTA kernel), else one buffer reused box after box.
    static constexpr int EPI_BOXES = EPI_FULL_BOXES + (EPI_REM > 0 ? 1 : 0);
    static constexpr int EPI_BUFS =
        1024 + EPI_OFFSET + NUM_WG * EPI_BOXES * EPI_WG_BYTES <= 232448 ? EPI_BOXES : 1;
    static constexpr int SMEM_BYTES = 1024 /*align slack*/ + EPI_OFFSET + NUM_WG * EPI_BUFS * EPI_WG_BYTES;

    static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "pair MMA N (M = 256): multiple of 32 up to 256");
    static_assert(BN % NUM_WG == 0 && NUM_WG >= 2 && NUM_WG <= 4, "promotion warpgroups");
    static_assert(!REBALANCE || (NUM_WG * 128 * PROMO_REGS + 128 * CTRL_REGS <= THREADS * LAUNCH_REGS &&
                                 LAUNCH_REGS % 8 == 0 && PROMO_REGS >= LAUNCH_REGS && CTRL_REGS <= LAUNCH_REGS),
                  "setmaxnreg budgets must fit the registers the block is launched with");
    static_assert(BN_WG % 8 == 0 && BN_WG <= 128, "promotion columns per warpgroup");
    static_assert(B_BYTES % 1024 == 0, "B tiles must keep 1024-byte swizzle atoms aligned");
    static_assert(NBUF >= 2, "double-buffered TMEM at least");
    static_assert(KS >= 1 && KS <= 4, "K blocks per stage");
    static_assert(EPI_REM % 8 == 0, "remainder box of whole 16-byte rows");
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

// A pair wait: as warp_wait_bounded, and a CTA that gives up also raises the
// abort flag of its peer, so the peer's waits end at once.
__device__ __forceinline__ bool pair_warp_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns,
                                               volatile int *abort_flag, uint32_t peer_abort,
                                               uint32_t role, uint32_t stage)
{
    int ok = 0;
    if ((threadIdx.x & 31) == 0) {
        ok = wait_bounded(bar, parity, timeout_ns, abort_flag, role, stage, true) ? 1 : 0;
        if (!ok)
            st_shared_cluster_u32(peer_abort, 1u);
    }
    return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

template <int BN, int STAGES, int KS, int LAYOUT, int NWG, bool REBAL = false>
__global__ void __launch_bounds__(PairConfig<BN, STAGES, KS, NWG, REBAL>::THREADS, 1)
    fp8_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                         const __grid_constant__ CUtensorMap tmap_b,
                         const __grid_constant__ CUtensorMap tmap_dbox,
                         const __grid_constant__ CUtensorMap tmap_drem, const GemmParams p)
{
    using Cfg = PairConfig<BN, STAGES, KS, NWG, REBAL>;
    constexpr int BN_WG = Cfg::BN_WG;
    constexpr int RMAX = Cfg::RMAX;
    constexpr int NBUF = Cfg::NBUF;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *a_tiles = smem;                               // [STAGES*KS][128][128 B]
    uint8_t *b_tiles = smem + STAGES * KS * Cfg::A_BYTES;  // [STAGES*KS][BN/2][128 B]
    float *sa_tiles = reinterpret_cast<float *>(smem + STAGES * Cfg::STAGE_BYTES);  // [STAGES*KS][128]
    float *sb_tiles = sa_tiles + STAGES * KS * kBM;        // [STAGES*KS][4]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sb_tiles + STAGES * KS * 4);
    uint64_t *full_bar = bars;                  // (leader) both CTAs' operand boxes landed
    uint64_t *sfull_bar = bars + STAGES;        // this CTA's scale copies landed
    uint64_t *empty_bar = bars + 2 * STAGES;    // pair MMAs of the stage done
    uint64_t *sread_bar = bars + 3 * STAGES;    // this CTA's promotion warps read the scales
    uint64_t *tfull_bar = bars + 4 * STAGES;    // TMEM partial buffer written
    uint64_t *tempty_bar = bars + 4 * STAGES + NBUF;  // (leader) both CTAs read the buffer
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4 * STAGES + 2 * NBUF);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    uint8_t *epi_stage = smem + Cfg::EPI_OFFSET;  // 1024-byte aligned, EPI_BUFS buffers per warpgroup

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    stamp_start(p);

    if (warp == Cfg::PRODUCER_A_WARP && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            // full: one expect-tx arrival from each of the leader's two
            // producers; the bytes of both CTAs' boxes
            mbar_init(smem_addr(full_bar + s), 2);
            // sfull: one cp.async arrival from each lane of the A producer
            mbar_init(smem_addr(sfull_bar + s), 32);
            mbar_init(smem_addr(empty_bar + s), 1);
            mbar_init(smem_addr(sread_bar + s), Cfg::NUM_PROMO_WARPS);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(smem_addr(tfull_bar + b), 1);
            mbar_init(smem_addr(tempty_bar + b), 2 * Cfg::NUM_PROMO_WARPS);
        }
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmap_a);
        tma_prefetch_desc(&tmap_b);
        if (Cfg::EPI_FULL_BOXES > 0)
            tma_prefetch_desc(&tmap_dbox);
        if (Cfg::EPI_REM > 0)
            tma_prefetch_desc(&tmap_drem);
    }
    if (warp == Cfg::MMA_WARP) {
        tmem_alloc_pair(smem_addr(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish_alloc_permit_pair();
    }
    tc_fence_before_sync();
    __syncthreads();
    // both CTAs' barriers exist before either signals the other
    cluster_sync();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    const uint64_t tmo = p.timeout_ns;
    const uint64_t drain_tmo = tmo > 1000000000ull ? tmo : 1000000000ull;
    const uint32_t peer_abort = map_shared_rank(smem_addr(const_cast<int *>(abort_flag)), rank ^ 1u);
    const uint32_t full_leader = map_shared_rank(smem_addr(full_bar), 0);
    const uint32_t tempty_leader = map_shared_rank(smem_addr(tempty_bar), 0);

    if (warp >= Cfg::NUM_PROMO_WARPS) {
    // The control warps.  With REBALANCE, the whole control warpgroup gives
    // registers up here, at one point that dominates all of its code.
    if constexpr (Cfg::REBALANCE)
        setmaxnreg_dec<Cfg::CTRL_REGS>();
    if (warp == Cfg::PRODUCER_A_WARP || warp == Cfg::PRODUCER_B_WARP) {
        // ------------------------------------------------------ TMA producers
        // Warp A: this CTA's A box per stage, plus cp.async copies of the
        // stage's LHS scales (each lane a 16-byte piece) and weight-block
        // scales (lanes 0-2).  Warp B: this CTA's half of the B box.
        const bool is_a = warp == Cfg::PRODUCER_A_WARP;
        PairScheduler<LAYOUT> sched(p);
        TileCoord tc;
        uint32_t stage = 0, phase = 0;
        // Test hook (dg_set_stall_injection): the first pair never fills a
        // stage, so its consumers' waits run out and report DG_ERR_TIMEOUT.
        bool ok = !(p.stall_injection && blockIdx.x < 2);
        while (ok && sched.next(tc, is_a && leader && lane == 0)) {
            const int m0 = tc.mb * kPairBM + static_cast<int>(rank) * kBM;  // this CTA's first row
            const int a_row = (LAYOUT == kMasked ? tc.g * p.M : 0) + m0;
            const int b_row = tc.g * p.N + tc.nb * BN + static_cast<int>(rank) * Cfg::BN_HALF;
            const float *sa_base = p.sA +
                                   (LAYOUT == kMasked ? static_cast<size_t>(tc.g) * p.num_kb * p.sa_ld : 0) +
                                   m0 + 4 * lane;
            const bool sa_lane_ok = m0 + 4 * lane < p.sa_ld;
            const int nb_first = (tc.nb * BN) / 128;
            const float *sb_src = p.sB + (static_cast<size_t>(tc.g) * p.nbn +
                                          min(nb_first + (lane < 3 ? lane : 0), p.nbn - 1)) * p.num_kb;
            for (int kb0 = 0; kb0 < p.num_kb; kb0 += KS) {
                if (!pair_warp_wait(smem_addr(empty_bar + stage), phase ^ 1, tmo, abort_flag, peer_abort,
                                    kRoleProducer, stage) ||
                    (is_a && !pair_warp_wait(smem_addr(sread_bar + stage), phase ^ 1, tmo, abort_flag,
                                             peer_abort, kRoleProducer, 64 + stage))) {
                    ok = false;
                    break;
                }
                const uint32_t fb = full_leader + 8 * stage;
                if (elect_one()) {
                    if (is_a) {
                        if (leader)
                            mbar_arrive_expect_tx(smem_addr(full_bar + stage), 2 * KS * Cfg::A_BYTES);
                        // dense: A rows are read again by the band's other
                        // column tiles while B streams past -- keep them in L2
                        if (LAYOUT == kDense)
                            tma_load_3d_pair_hint(smem_addr(a_tiles + stage * KS * Cfg::A_BYTES), &tmap_a, fb,
                                                  0, a_row, kb0, l2_policy_evict_last());
                        else
                            tma_load_3d_pair(smem_addr(a_tiles + stage * KS * Cfg::A_BYTES), &tmap_a, fb, 0,
                                             a_row, kb0);
                    } else {
                        if (leader)
                            mbar_arrive_expect_tx(smem_addr(full_bar + stage), 2 * KS * Cfg::B_BYTES);
                        tma_load_3d_pair(smem_addr(b_tiles + stage * KS * Cfg::B_BYTES), &tmap_b, fb, 0,
                                         b_row, kb0);
                    }
                }
                if (is_a) {
#pragma unroll
                    for (int q = 0; q < KS; ++q) {
                        const int kb = kb0 + q;
                        const bool in_k = kb < p.num_kb;
                        const bool sa_ok = in_k && sa_lane_ok;
                        cp_async_16(smem_addr(sa_tiles + (stage * KS + q) * kBM) + 16 * lane,
                                    sa_ok ? static_cast<const void *>(sa_base + static_cast<size_t>(kb) * p.sa_ld)
                                          : static_cast<const void *>(p.sA),
                                    sa_ok ? 16u : 0u);
                        if (lane < 3)
                            cp_async_4(smem_addr(sb_tiles + (stage * KS + q) * 4) + 4 * lane,
                                       sb_src + (in_k ? kb : p.num_kb - 1));
                    }
                    cp_async_mbar_arrive_noinc(smem_addr(sfull_bar + stage));
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        if (is_a)
            cp_async_wait_all();
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
    } else if (warp == Cfg::MMA_WARP) {
        // ------------------------------------------------ MMA issuer (leader)
        if (leader) {
            PairScheduler<LAYOUT> sched(p);
            TileCoord tc;
            uint32_t stage = 0, phase = 0, acc_i = 0;
            uint32_t last_bar = 0, last_parity = 0;  // most recent commit
            bool ok = true;
            constexpr uint32_t idesc = idesc_e4m3_f32(kPairBM, BN);
            const uint64_t a_desc0 = smem_desc_k_sw128(smem_addr(a_tiles));
            const uint64_t b_desc0 = smem_desc_k_sw128(smem_addr(b_tiles));
            while (ok && sched.next(tc, false)) {
                for (int kb0 = 0; kb0 < p.num_kb; kb0 += KS) {
                    if (!pair_warp_wait(smem_addr(full_bar + stage), phase, tmo, abort_flag, peer_abort,
                                        kRoleMma, stage)) {
                        ok = false;
                        break;
                    }
#pragma unroll
                    for (int q = 0; q < KS; ++q) {
                        if (kb0 + q >= p.num_kb)
                            break;
                        const uint32_t buf = acc_i % NBUF, tph = (acc_i / NBUF) & 1;
                        if (!pair_warp_wait(smem_addr(tempty_bar + buf), tph ^ 1, tmo, abort_flag,
                                            peer_abort, kRoleMma, 16 + buf)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        const uint32_t d_tmem = tmem_base + buf * Cfg::ACC_STRIDE;
                        const uint64_t ad = a_desc0 + static_cast<uint64_t>(((stage * KS + q) * Cfg::A_BYTES) >> 4);
                        const uint64_t bd = b_desc0 + static_cast<uint64_t>(((stage * KS + q) * Cfg::B_BYTES) >> 4);
                        if (elect_one()) {
#pragma unroll
                            for (int j = 0; j < kBK / 32; ++j)
                                mma_f8f6f4_pair(d_tmem, ad + 2 * j, bd + 2 * j, idesc, j > 0 ? 1u : 0u);
                            mma_commit_pair_multicast(smem_addr(tfull_bar + buf), 0x3);
                        }
                        __syncwarp();
                        last_bar = smem_addr(tfull_bar + buf);
                        last_parity = tph;
                        ++acc_i;
                    }
                    if (!ok)
                        break;
                    if (elect_one())
                        mma_commit_pair_multicast(smem_addr(empty_bar + stage), 0x3);
                    __syncwarp();
                    last_bar = smem_addr(empty_bar + stage);
                    last_parity = phase;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // Drain: every pair MMA issued here has finished once the most
            // recent commit has fired.
            if (lane == 0 && last_bar != 0)
                wait_bounded(last_bar, last_parity, drain_tmo, abort_flag, kRoleDrain, 32, false);
            __syncwarp();
        }
    }
    } else {
        // ------------------------------------------------ promotion warps
        if constexpr (Cfg::REBALANCE)
            setmaxnreg_inc<Cfg::PROMO_REGS>();
        const int wg = warp / 4;
        const int quad = warp % 4;
        const int row = quad * 32 + lane;  // row within this CTA's half == TMEM lane
        const int wg_tid = threadIdx.x % 128;
        const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
        PairScheduler<LAYOUT> sched(p);
        TileCoord tc;
        uint32_t acc_i = 0, stage = 0, phase = 0;
        bool ok = true;
        float acc[BN_WG];

        while (ok && sched.next(tc, false)) {
            const int m_half = tc.mb * kPairBM + static_cast<int>(rank) * kBM;  // first row of this half
            const int m_local = m_half + row;  // row index inside the group
            bool row_ok;
            if constexpr (LAYOUT == kDense) {
                row_ok = m_local < p.M;
            } else if constexpr (LAYOUT == kContiguous) {
                row_ok = false;
                // a row is computed when its index is this visit's group and
                // the group of its own 128-row block (the group of the
                // block's first row)
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
            const int col0 = tc.nb * BN + wg * BN_WG;  // first column of this warpgroup
            const int nb_first = (tc.nb * BN) / 128;
            const int nb_lo = min(col0 / 128, p.nbn - 1);
            const int j_lo = nb_lo - nb_first;
            const int j_hi = min(nb_lo + 1, p.nbn - 1) - nb_first;
            const int boundary = (nb_lo + 1) * 128 - col0;  // local column where sB switches
#pragma unroll
            for (int i = 0; i < BN_WG; ++i)
                acc[i] = 0.0f;

            for (int kb0 = 0; kb0 < p.num_kb; kb0 += KS) {
                if (!pair_warp_wait(smem_addr(sfull_bar + stage), phase, tmo, abort_flag, peer_abort,
                                    kRolePromote, stage)) {
                    ok = false;
                    break;
                }
                float s_lo[KS], s_hi[KS];
#pragma unroll
                for (int q = 0; q < KS; ++q) {
                    const float sa = sa_tiles[(stage * KS + q) * kBM + row];
                    s_lo[q] = sa * sb_tiles[(stage * KS + q) * 4 + j_lo];
                    s_hi[q] = sa * sb_tiles[(stage * KS + q) * 4 + j_hi];
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(smem_addr(sread_bar + stage));
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
#pragma unroll
                for (int q = 0; q < KS; ++q) {
                    if (kb0 + q >= p.num_kb)
                        break;
                    const uint32_t buf = acc_i % NBUF, tph = (acc_i / NBUF) & 1;
                    if (!pair_warp_wait(smem_addr(tfull_bar + buf), tph, tmo, abort_flag, peer_abort,
                                        kRolePromote, 16 + buf)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t taddr = tmem_base + lane_bits + buf * Cfg::ACC_STRIDE + wg * BN_WG;
#pragma unroll
                    for (int c0 = 0; c0 < BN_WG; c0 += RMAX) {
                        constexpr int TAIL = BN_WG % RMAX;
                        uint32_t r[RMAX];
                        const bool whole = c0 + RMAX <= BN_WG;
                        if (whole)
                            tmem_load_cols<RMAX>(taddr + c0, r);
                        else
                            tmem_load_cols<TAIL>(taddr + c0, r);
                        tmem_ld_wait();
                        if (c0 + RMAX >= BN_WG) {
                            // every column of this buffer is in registers:
                            // hand it back to the leader's MMA warp
                            tc_fence_before_sync();
                            __syncwarp();
                            if (lane == 0)
                                mbar_arrive_cluster(tempty_leader + 8 * buf);
                        }
#pragma unroll
                        for (int g8 = 0; g8 < RMAX; g8 += 8) {
                            if (whole || g8 < TAIL) {
                                // a warpgroup whose columns never straddle a
                                // 128-wide weight block uses one scale
                                const float sc = (Cfg::UNIFORM_SCALE || c0 + g8 < boundary) ? s_lo[q] : s_hi[q];
#pragma unroll
                                for (int i = 0; i < 8; i += 2)
                                    fma2_rn(acc[c0 + g8 + i], acc[c0 + g8 + i + 1], __uint_as_float(r[g8 + i]),
                                            __uint_as_float(r[g8 + i + 1]), sc);
                            }
                        }
                    }
                    ++acc_i;
                }
                if (!ok)
                    break;
            }

            // ------------------------------------------------------ epilogue
            // As in the one-CTA kernel: whole-box TMA stores when every row of
            // the warpgroup may be written, row-wise stores otherwise; a warp
            // that gave up still joins the first barrier and the warpgroup
            // leaves together.
            if (!named_barrier_and(1 + wg, 128, ok)) {
                ok = false;
                break;
            }
            if constexpr (LAYOUT == kDense) {
                if (p.D32) {
                    // accumulate form: fp32 C + acc, row by row
                    if (row_ok)
                        store_row_acc_f32<BN_WG>(p.C + static_cast<size_t>(m_local) * p.N + col0,
                                                 p.D32 + static_cast<size_t>(m_local) * p.N + col0, acc, col0,
                                                 p.N);
                    continue;
                }
            }
            const bool tile_rows_ok = named_barrier_and(
                1 + wg, 128, LAYOUT == kDense ? (m_half < p.M) : row_ok);
            if (tile_rows_ok) {
                const int grow0 = (LAYOUT == kMasked ? tc.g * p.M : 0) + m_half;
#pragma unroll
                for (int bx = 0; bx < Cfg::EPI_BOXES; ++bx) {
                    const bool full = bx < Cfg::EPI_FULL_BOXES;
                    const int cbase = bx * Cfg::EPI_BOX;
                    const int ncols = full ? Cfg::EPI_BOX : Cfg::EPI_REM;
                    if (col0 + cbase >= p.N)
                        break;  // this box (and any after it) lies past N
                    const uint32_t stg =
                        smem_addr(epi_stage + (wg * Cfg::EPI_BUFS + bx % Cfg::EPI_BUFS) * Cfg::EPI_WG_BYTES);
                    if (wg_tid == 0)
                        bulk_wait_group_read<Cfg::EPI_BUFS - 1>();
                    named_barrier_sync(1 + wg, 128);
#pragma unroll
                    for (int ch = 0; ch < Cfg::EPI_BOX / 8; ++ch) {
                        if (ch * 8 < ncols) {
                            // full boxes: 64-byte rows, 16-byte chunk index
                            // XOR ((row / 2) % 4) (64-byte swizzle);
                            // remainder: dense rows of ncols * 2 bytes
                            const uint32_t off =
                                full ? static_cast<uint32_t>(row * 64 + ((ch ^ ((row >> 1) & 3)) * 16))
                                     : static_cast<uint32_t>(row * ncols * 2 + ch * 16);
                            st_shared_v4(stg + off, pack_bf16x8(acc + cbase + ch * 8));
                        }
                    }
                    fence_proxy_async_smem();
                    named_barrier_sync(1 + wg, 128);
                    if (wg_tid == 0) {
                        tma_store_2d(full ? static_cast<const void *>(&tmap_dbox)
                                          : static_cast<const void *>(&tmap_drem),
                                     stg, col0 + cbase, grow0);
                        bulk_commit_group();
                    }
                }
            } else if (row_ok) {
                const size_t grow = (LAYOUT == kMasked ? static_cast<size_t>(tc.g) * p.M : 0) +
                                    static_cast<size_t>(m_local);
                __nv_bfloat16 *drow = p.D + grow * p.N + col0;
#pragma unroll
                for (int c = 0; c < BN_WG; c += 8)
                    if (col0 + c < p.N)
                        *reinterpret_cast<uint4 *>(drow + c) = pack_bf16x8(acc + c);
            }
        }
        if (wg_tid == 0)
            bulk_wait_group<0>();
        __syncwarp();
    }

    __syncthreads();
    // no CTA leaves (or frees TMEM) while its peer may still signal its
    // barriers or the leader's MMAs may still write its TMEM
    cluster_sync();
    stamp_end(p);
    if (warp == Cfg::MMA_WARP) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace dg
