// fp8_gemm_kernel.cuh -- persistent, warp-specialised sm_100a kernel for the
// fine-grained-scaled FP8 GEMM (dense, contiguous-grouped, masked-grouped).
//
// Method (DeepGEMM pages): each 128-wide K block is contracted on the tensor
// cores and its partial promoted on the CUDA cores into an fp32 accumulator,
// acc += (sA[m,kb] * sB[n/128,kb]) * partial  (DeepGEMM article, lqnn.cn,
// section "DeepGEMM", two-level accumulation; pxiaoer.blog analysis, section
// "DeepGEMM介绍").  Persistent warp specialisation overlaps data movement,
// MMA and promotion (lqnn.cn article, section "持久化线程束专用化"); one block
// scheduler serves the dense and both grouped layouts (section
// "统一且经过优化的块调度器"); tile shapes, stages and layouts are
// compile-time constants (section "完全JIT设计").
//
// B200 design of one CTA (one per SM, persistent over tiles of 128 x BN):
//   warp P (producer)  : TMA loads of the A tile (128 x 128 e4m3) and the
//                        B tile (BN x 128 e4m3) of each K block into a
//                        STAGES-deep shared-memory ring (mbarrier full/empty).
//   warp M (MMA)       : 4 x tcgen05.mma kind::f8f6f4 (K = 32 each) per K
//                        block into one of two TMEM partial buffers, then
//                        tcgen05.commit to free the smem stage and to hand
//                        the partial to the promotion warps.
//   promotion warps    : 1 or 2 warpgroups (BN <= 128: one; otherwise two,
//                        splitting the columns).  Thread t of a warpgroup owns
//                        tile row t (= TMEM lane t).  Per K block it loads its
//                        row's partial from TMEM, frees the buffer, and does
//                        acc = fma(partial, sA*sB, acc) in registers.  The
//                        scales are read with plain (cached) loads one block
//                        ahead.  After the last block it rounds to bf16 and
//                        stores its row segment.
// The MMA of block kb+1 runs while block kb is being promoted (double TMEM),
// and the next tile's first MMAs run under the previous tile's epilogue.
//
// Every mbarrier wait is bounded in time: on expiry the waiting role records
// DG_ERR_TIMEOUT (role, stage, CTA) in the device status word, raises a
// CTA-wide abort flag, and all roles leave their loops; the producer and the
// MMA warp then wait (bounded) for their in-flight copies and MMAs, and TMEM
// is freed before the CTA exits.  Nothing traps.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "ptx_sm100.cuh"

namespace dg {

enum Layout : int { kDense = 0, kContiguous = 1, kMasked = 2 };

// Device status word: code (bits 0-7), role (8-11), stage (12-19), CTA (20-31).
constexpr uint32_t kCodeTimeout = 5;
constexpr uint32_t kCodeBadGroup = 6;
enum Role : uint32_t { kRoleProducer = 1, kRoleMma = 2, kRolePromote = 3, kRoleDrain = 4, kRoleSched = 5 };

static __device__ unsigned int g_status_word = 0;

__device__ __forceinline__ void record_status(uint32_t code, uint32_t role, uint32_t stage)
{
    const uint32_t w = (code & 0xFF) | ((role & 0xF) << 8) | ((stage & 0xFF) << 12) |
                       ((blockIdx.x & 0xFFF) << 20);
    atomicCAS(&g_status_word, 0u, w);
}

struct GemmParams {
    const float *sA;          // dense/contig: [K/128][sa_ld]; masked: [G][K/128][sa_ld]
    const float *sB;          // [G][nbn][K/128]
    __nv_bfloat16 *D;         // dense/contig: [M][N]; masked: [G][M][N]
    const int32_t *m_indices; // contiguous only
    const int32_t *masked_m;  // masked only
    int M;                    // dense: M; contiguous: M_total; masked: max_m
    int N, K, G;
    int sa_ld;                // padded row count of the transposed LHS scales
    int num_kb;               // K / 128
    int nbn;                  // ceil(N / 128)
    int num_mb;               // dense/contig: ceil(M / 128)
    int num_nb;               // ceil(N / BN)
    int raster;               // m-blocks per rasterisation group (dense/contig)
    unsigned long long timeout_ns;
};

constexpr int kBM = 128;
constexpr int kBK = 128;

// ---------------------------------------------------------------- scheduler

struct TileCoord {
    int g, mb, nb;
};

// Enumerates this CTA's tiles: t = blockIdx.x, blockIdx.x + gridDim.x, ...
// Every role runs its own copy and sees the same sequence.
template <int LAYOUT>
struct TileScheduler {
    const GemmParams &p;
    int next_t;
    int cur_g = 0, cur_base = 0, cur_count = -1;

    __device__ explicit TileScheduler(const GemmParams &params) : p(params), next_t(blockIdx.x) {}

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
                    cur_count = ((mm + kBM - 1) / kBM) * p.num_nb;
                }
                if (t < cur_base + cur_count)
                    break;
                cur_base += cur_count;
                ++cur_g;
                cur_count = -1;
            }
            next_t += gridDim.x;
            const int local = t - cur_base;
            const int mbs = cur_count / p.num_nb;
            tc.g = cur_g;
            tc.nb = local / mbs;
            tc.mb = local - tc.nb * mbs;
            return true;
        } else {
            const int total = p.num_mb * p.num_nb;
            while (next_t < total) {
                const int t = next_t;
                next_t += gridDim.x;
                const int per = p.raster * p.num_nb;
                const int grp = t / per;
                const int within = t - grp * per;
                const int rows_here = min(p.raster, p.num_mb - grp * p.raster);
                tc.mb = grp * p.raster + within % rows_here;
                tc.nb = within / rows_here;
                tc.g = 0;
                if constexpr (LAYOUT == kContiguous) {
                    const int g = __ldg(p.m_indices + tc.mb * kBM);
                    if (g < 0)
                        continue;  // padding block: rows stay untouched
                    if (g >= p.G) {
                        if (report)
                            record_status(kCodeBadGroup, kRoleSched, 0);
                        continue;
                    }
                    tc.g = g;
                }
                return true;
            }
            return false;
        }
    }
};

// ----------------------------------------------------------- bounded waits

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, uint64_t timeout_ns,
                                             volatile int *abort_flag, uint32_t role,
                                             uint32_t stage, bool honour_abort)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    uint32_t spins = 0;
    while (true) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((++spins & 63u) == 0) {
            if (honour_abort && *abort_flag)
                return false;
            if (global_timer_ns() - t0 > timeout_ns) {
                *abort_flag = 1;
                record_status(kCodeTimeout, role, stage);
                return false;
            }
        }
    }
}

// Lane 0 waits, the whole warp gets the outcome.
__device__ __forceinline__ bool warp_wait_bounded(uint32_t bar, uint32_t parity,
                                                  uint64_t timeout_ns, volatile int *abort_flag,
                                                  uint32_t role, uint32_t stage)
{
    int ok = 0;
    if ((threadIdx.x & 31) == 0)
        ok = wait_bounded(bar, parity, timeout_ns, abort_flag, role, stage, true) ? 1 : 0;
    return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

// ------------------------------------------------------------------ config

template <int BN_, int STAGES_>
struct KernelConfig {
    static constexpr int BN = BN_;
    static constexpr int STAGES = STAGES_;
    static constexpr int NUM_WG = BN > 128 ? 2 : 1;
    static constexpr int BN_WG = BN / NUM_WG;
    static constexpr int NUM_PROMO_WARPS = 4 * NUM_WG;
    static constexpr int PRODUCER_WARP = NUM_PROMO_WARPS;
    static constexpr int MMA_WARP = NUM_PROMO_WARPS + 1;
    static constexpr int THREADS = (NUM_PROMO_WARPS + 2) * 32;
    static constexpr int A_BYTES = kBM * kBK;
    static constexpr int B_BYTES = BN * kBK;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int ACC_STRIDE = BN <= 128 ? 128 : 256;  // TMEM columns per buffer
    static constexpr int TMEM_COLS = 2 * ACC_STRIDE;
    static constexpr int BAR_BYTES = 8 * (2 * STAGES + 4) + 16;
    static constexpr int SMEM_BYTES = 1024 /*align slack*/ + STAGES * STAGE_BYTES + BAR_BYTES;

    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128: multiple of 16, <= 256");
    static_assert(BN_WG % 16 == 0, "promotion columns per warpgroup must be a multiple of 16");
    static_assert(BN_WG <= 128, "a warpgroup's column range must fit one 128-wide sB block pair");
    static_assert(B_BYTES % 1024 == 0, "B stage must keep 1024-byte swizzle atoms aligned");
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

// ------------------------------------------------------------------ kernel

template <int BN, int STAGES, int LAYOUT>
__global__ void __launch_bounds__(KernelConfig<BN, STAGES>::THREADS, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                    const __grid_constant__ CUtensorMap tmap_b, const GemmParams p)
{
    using Cfg = KernelConfig<BN, STAGES>;
    constexpr int BN_WG = Cfg::BN_WG;
    constexpr int CHUNKS = BN_WG / 16;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *a_tiles = smem;
    uint8_t *b_tiles = smem + STAGES * Cfg::A_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * Cfg::STAGE_BYTES);
    uint64_t *full_bar = bars;
    uint64_t *empty_bar = bars + STAGES;
    uint64_t *tfull_bar = bars + 2 * STAGES;
    uint64_t *tempty_bar = bars + 2 * STAGES + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    if (warp == Cfg::PRODUCER_WARP && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_addr(full_bar + s), 1);
            mbar_init(smem_addr(empty_bar + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_addr(tfull_bar + b), 1);
            mbar_init(smem_addr(tempty_bar + b), Cfg::NUM_PROMO_WARPS);
        }
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmap_a);
        tma_prefetch_desc(&tmap_b);
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

    if (warp == Cfg::PRODUCER_WARP) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            TileScheduler<LAYOUT> sched(p);
            TileCoord tc;
            uint32_t stage = 0, phase = 0;
            uint32_t issued = 0;
            bool ok = true;
            while (ok && sched.next(tc, true)) {
                const int a_row = (LAYOUT == kMasked ? tc.g * p.M : 0) + tc.mb * kBM;
                const int b_row = tc.g * p.N + tc.nb * BN;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!wait_bounded(smem_addr(empty_bar + stage), phase ^ 1, tmo, abort_flag,
                                      kRoleProducer, stage, true)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_addr(full_bar + stage);
                    mbar_arrive_expect_tx(fb, Cfg::STAGE_BYTES);
                    tma_load_2d(smem_addr(a_tiles + stage * Cfg::A_BYTES), &tmap_a, fb, kb * kBK,
                                a_row);
                    tma_load_2d(smem_addr(b_tiles + stage * Cfg::B_BYTES), &tmap_b, fb, kb * kBK,
                                b_row);
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // Drain: the last min(STAGES, issued) loads must have landed
            // before the CTA may exit (always true on the normal path).
            const uint32_t first = issued > STAGES ? issued - STAGES : 0;
            for (uint32_t i = first; i < issued; ++i)
                wait_bounded(smem_addr(full_bar + i % STAGES), (i / STAGES) & 1, tmo, abort_flag,
                             kRoleDrain, i % STAGES, false);
        }
        __syncwarp();
    } else if (warp == Cfg::MMA_WARP) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            TileScheduler<LAYOUT> sched(p);
            TileCoord tc;
            uint32_t stage = 0, phase = 0, acc_i = 0, committed = 0;
            bool ok = true;
            constexpr uint32_t idesc = idesc_e4m3_f32(kBM, BN);
            while (ok && sched.next(tc, false)) {
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    const uint32_t buf = acc_i & 1, tph = (acc_i >> 1) & 1;
                    if (!wait_bounded(smem_addr(tempty_bar + buf), tph ^ 1, tmo, abort_flag,
                                      kRoleMma, 16 + buf, true) ||
                        !wait_bounded(smem_addr(full_bar + stage), phase, tmo, abort_flag,
                                      kRoleMma, stage, true)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t d_tmem = tmem_base + buf * Cfg::ACC_STRIDE;
                    const uint32_t a0 = smem_addr(a_tiles + stage * Cfg::A_BYTES);
                    const uint32_t b0 = smem_addr(b_tiles + stage * Cfg::B_BYTES);
#pragma unroll
                    for (int j = 0; j < kBK / 32; ++j)
                        mma_f8f6f4(d_tmem, smem_desc_k_sw128(a0 + j * 32),
                                   smem_desc_k_sw128(b0 + j * 32), idesc, j > 0 ? 1u : 0u);
                    mma_commit(smem_addr(empty_bar + stage));
                    mma_commit(smem_addr(tfull_bar + buf));
                    ++committed;
                    ++acc_i;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // Drain: the last commit (to the empty barrier of the last stage
            // used) fires once every MMA issued by this thread has finished.
            if (committed > 0) {
                const uint32_t i = committed - 1;
                wait_bounded(smem_addr(empty_bar + i % STAGES), (i / STAGES) & 1, tmo, abort_flag,
                             kRoleDrain, 32 + i % STAGES, false);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ promotion warps
        const int wg = warp / 4;
        const int quad = warp % 4;
        const int row = quad * 32 + lane;  // tile row == TMEM lane
        const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
        TileScheduler<LAYOUT> sched(p);
        TileCoord tc;
        uint32_t acc_i = 0;
        bool ok = true;
        float acc[BN_WG];

        while (ok && sched.next(tc, false)) {
            const int m_local = tc.mb * kBM + row;  // row index inside the group
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
            const float *sa_ptr = p.sA +
                                  (LAYOUT == kMasked ? static_cast<size_t>(tc.g) * p.num_kb * p.sa_ld
                                                     : 0) +
                                  m_local;
            const int col0 = tc.nb * BN + wg * BN_WG;  // first column of this warpgroup
            const int nb_lo = min(col0 / 128, p.nbn - 1);
            const int nb_hi = min(nb_lo + 1, p.nbn - 1);
            const int boundary = (nb_lo + 1) * 128 - col0;  // local column where sB switches
            const float *sb_lo = p.sB + (static_cast<size_t>(tc.g) * p.nbn + nb_lo) * p.num_kb;
            const float *sb_hi = p.sB + (static_cast<size_t>(tc.g) * p.nbn + nb_hi) * p.num_kb;

            float sa_next = row_ok ? __ldg(sa_ptr) : 0.0f;
            float sbl_next = __ldg(sb_lo);
            float sbh_next = __ldg(sb_hi);
#pragma unroll
            for (int i = 0; i < BN_WG; ++i)
                acc[i] = 0.0f;

            for (int kb = 0; kb < p.num_kb; ++kb) {
                const float sa = sa_next, sbl = sbl_next, sbh = sbh_next;
                if (kb + 1 < p.num_kb) {
                    sa_next = row_ok ? __ldg(sa_ptr + static_cast<size_t>(kb + 1) * p.sa_ld) : 0.0f;
                    sbl_next = __ldg(sb_lo + kb + 1);
                    sbh_next = __ldg(sb_hi + kb + 1);
                }
                const float s_lo = sa * sbl;
                const float s_hi = sa * sbh;
                const uint32_t buf = acc_i & 1, tph = (acc_i >> 1) & 1;
                if (!warp_wait_bounded(smem_addr(tfull_bar + buf), tph, tmo, abort_flag,
                                       kRolePromote, 16 + buf)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t taddr = tmem_base + lane_bits + buf * Cfg::ACC_STRIDE + wg * BN_WG;
#pragma unroll
                for (int c = 0; c < CHUNKS; c += 2) {
                    uint32_t r0[16], r1[16];
                    tmem_ld_32x32b_x16(taddr + c * 16, r0);
                    if (c + 1 < CHUNKS)
                        tmem_ld_32x32b_x16(taddr + (c + 1) * 16, r1);
                    tmem_ld_wait();
                    if (c + 2 >= CHUNKS) {
                        // every column of this buffer is in registers: free it
                        tc_fence_before_sync();
                        __syncwarp();
                        if (lane == 0)
                            mbar_arrive(smem_addr(tempty_bar + buf));
                    }
                    const float s0 = (c * 16 >= boundary) ? s_hi : s_lo;
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        acc[c * 16 + i] = fmaf(__uint_as_float(r0[i]), s0, acc[c * 16 + i]);
                    if (c + 1 < CHUNKS) {
                        const float s1 = ((c + 1) * 16 >= boundary) ? s_hi : s_lo;
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            acc[(c + 1) * 16 + i] =
                                fmaf(__uint_as_float(r1[i]), s1, acc[(c + 1) * 16 + i]);
                    }
                }
                ++acc_i;
            }
            if (!ok)
                break;

            // ------------------------------------------------------ epilogue
            if (row_ok) {
                const size_t grow = (LAYOUT == kMasked ? static_cast<size_t>(tc.g) * p.M : 0) +
                                    static_cast<size_t>(m_local);
                __nv_bfloat16 *drow = p.D + grow * p.N + col0;
#pragma unroll
                for (int c = 0; c < BN_WG; c += 8) {
                    if (col0 + c < p.N) {
                        __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[c + 0], acc[c + 1]);
                        __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[c + 2], acc[c + 3]);
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[c + 4], acc[c + 5]);
                        __nv_bfloat162 h3 = __floats2bfloat162_rn(acc[c + 6], acc[c + 7]);
                        uint4 v;
                        v.x = *reinterpret_cast<uint32_t *>(&h0);
                        v.y = *reinterpret_cast<uint32_t *>(&h1);
                        v.z = *reinterpret_cast<uint32_t *>(&h2);
                        v.w = *reinterpret_cast<uint32_t *>(&h3);
                        *reinterpret_cast<uint4 *>(drow + c) = v;
                    }
                }
            }
        }
    }

    __syncthreads();
    if (warp == Cfg::MMA_WARP) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace dg
