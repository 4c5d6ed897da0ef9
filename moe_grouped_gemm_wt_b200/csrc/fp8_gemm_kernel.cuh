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
//   warp P (producer)  : per stage of KS K blocks, one 3-D TMA box of A
//                        (KS x 128 x 128 e4m3) and one of B (KS x BN x 128),
//                        plus cp.async copies of the 128 LHS scales and the
//                        (at most three) weight-block scales of each K block,
//                        into a STAGES-deep shared-memory ring; all land on
//                        the stage's "full" mbarrier (lqnn.cn article,
//                        section "Hopper TMA特性": TMA for the operands; the
//                        scales take the LSU path because each TMA
//                        instruction costs the SM's TMA engine a roughly
//                        fixed time, whatever its size).  With PROD2 (the
//                        masked layout's decode tile) a second warp issues
//                        the B boxes, in parallel with the A boxes.
//   warp M (MMA)       : 4 x tcgen05.mma kind::f8f6f4 (K = 32 each) per K
//                        block into one of NBUF (2..4) TMEM partial buffers,
//                        issued by one elected lane of a warp-uniform loop
//                        so the descriptors stay uniform, then
//                        tcgen05.commit to free the smem stage and to hand
//                        the partial to the promotion warps.
//   promotion warps    : two warpgroups splitting the tile's columns.
//                        Thread t of a warpgroup owns tile row t (= TMEM
//                        lane t).  Per K block it loads its row's partial
//                        from TMEM, frees the buffer, and does
//                        acc = fma(partial, sA*sB, acc) in registers, with
//                        the scales read from the stage in shared memory
//                        (released through a per-stage "scales read"
//                        barrier, since the MMA frees the operand tiles
//                        earlier).  After the last block it rounds to bf16
//                        and stores its row segment.
// The MMAs of blocks kb+1 .. kb+NBUF-1 run while block kb is being promoted,
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

// kKGrouped: the K-grouped TN GEMM (MoE weight gradient): groups own
// 128-row segments of the shared K axis, D is fp32 [G][M][N].
enum Layout : int { kDense = 0, kContiguous = 1, kMasked = 2, kKGrouped = 3 };

// Device status word: code (bits 0-7), role (8-11), stage (12-19), CTA (20-31).
constexpr uint32_t kCodeTimeout = 5;
constexpr uint32_t kCodeBadGroup = 6;
constexpr uint32_t kCodeBadScale = 8;
enum Role : uint32_t { kRoleProducer = 1, kRoleMma = 2, kRolePromote = 3, kRoleDrain = 4, kRoleSched = 5,
                       kRoleTransform = 6 };

static __device__ unsigned int g_status_word = 0;

__device__ __forceinline__ void record_status(uint32_t code, uint32_t role, uint32_t stage)
{
    // the CTA's linear index (the K-split kernels run a 3-D grid)
    const uint32_t cta = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
    const uint32_t w = (code & 0xFF) | ((role & 0xF) << 8) | ((stage & 0xFF) << 12) | ((cta & 0xFFF) << 20);
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
    int ksplit;               // CTAs of a cluster sharing one tile's K range (1 = no split)
    int kb_per_split;         // K blocks per split
    float *ws;                // K split: fp32 partials [tile][split][BN/4][128][4]
    int stall_injection;      // test hook: CTA 0's producer issues nothing
    unsigned long long timeout_ns;
    // Dense accumulate form D = C + A.B^T: when D32 is set the output is
    // fp32 D32[M][N] = C[M][N] + acc (C may be D32 itself) instead of bf16 D.
    const float *C;
    float *D32;
    const int32_t *k_offsets;  // K-grouped only: [G+1] K-row offsets of the groups
    // UE8M0 block-scaled mode: packed scales, four K blocks per int32.
    const int32_t *sfa;  // dense/contig: [num_kg][sfa_ld]; masked: [G][num_kg][sfa_ld]
    const int32_t *sfb;  // [G][num_kg][nbn]
    int sfa_ld;          // padded row count of the packed LHS scales
    int num_kg;          // ceil(num_kb / 4)
    // Launch timing (dg_set_timing_stamps): when set, stamps[0] takes the
    // earliest CTA start and stamps[1] the latest CTA end (%globaltimer, ns).
    unsigned long long *stamps;
};

// Launch-timing stamps: thread 0 of each CTA folds its start and end time
// into the caller's pair (atomicMin / atomicMax, one each per CTA).
__device__ __forceinline__ void stamp_start(const GemmParams &p)
{
    if (p.stamps != nullptr && threadIdx.x == 0)
        atomicMin(p.stamps, static_cast<unsigned long long>(global_timer_ns()));
}
__device__ __forceinline__ void stamp_end(const GemmParams &p)
{
    if (p.stamps != nullptr) {
        __syncthreads();
        if (threadIdx.x == 0)
            atomicMax(p.stamps + 1, static_cast<unsigned long long>(global_timer_ns()));
    }
}

// Row segment of an fp32 output: drow[c] = acc[c] for the 4-float groups of
// this thread's row that lie inside N.
template <int COLS>
__device__ __forceinline__ void store_row_f32(float *drow, const float *acc, int col0, int N)
{
#pragma unroll
    for (int c = 0; c < COLS; c += 4)
        if (col0 + c < N)
            *reinterpret_cast<float4 *>(drow + c) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
}

// Row segment of the accumulate form: drow[c] = crow[c] + acc[c] for the
// 4-float groups of this thread's row that lie inside N (read before write,
// so crow == drow is fine).
template <int COLS>
__device__ __forceinline__ void store_row_acc_f32(const float *crow, float *drow, const float *acc, int col0,
                                                  int N)
{
#pragma unroll
    for (int c = 0; c < COLS; c += 4) {
        if (col0 + c < N) {
            const float4 cv = *reinterpret_cast<const float4 *>(crow + c);
            *reinterpret_cast<float4 *>(drow + c) =
                make_float4(cv.x + acc[c], cv.y + acc[c + 1], cv.z + acc[c + 2], cv.w + acc[c + 3]);
        }
    }
}

constexpr int kBM = 128;
constexpr int kBK = 128;

// ---------------------------------------------------------------- scheduler

struct TileCoord {
    int g, mb, nb;
};

// Contiguous layout: the segments are aligned to the 128-row M block, so a
// block whose first row is padding must hold padding only.  True when any
// row of the block [row0, row0 + 128) carries a group index (a malformed
// block: it is skipped and its rows stay untouched, but it is flagged).
// Run by one thread, only for blocks whose first row is padding.
__device__ __forceinline__ bool padding_block_has_rows(const int32_t *m_indices, int row0)
{
    int any = 0;
#pragma unroll 8
    for (int r = 1; r < kBM; ++r)
        any |= __ldg(m_indices + row0 + r) >= 0 ? 1 : 0;
    return any != 0;
}

// Enumerates this CTA's tiles: t = blockIdx.x, blockIdx.x + gridDim.x, ...
// Every role runs its own copy and sees the same sequence.  With SPLIT (the
// K-split kernels) the grid is 3-D -- x the split (a cluster of ksplit CTAs
// along x), y the column tile, z the 128-row block -- and each CTA has
// exactly one tile, so no index needs a division.
template <int LAYOUT, bool SPLIT = false>
struct TileScheduler {
    const GemmParams &p;
    int next_t;
    int cur_g = 0, cur_base = 0, cur_count = -1;

    int stride;

    __device__ explicit TileScheduler(const GemmParams &params)
        : p(params), next_t(SPLIT ? 0 : static_cast<int>(blockIdx.x)), stride(SPLIT ? 1 : static_cast<int>(gridDim.x)) {}

    // This CTA's K blocks: [begin, end).
    __device__ int kb_begin() const
    {
        if constexpr (LAYOUT == kKGrouped)
            return cur_kb0;
        return SPLIT ? static_cast<int>(blockIdx.x) * p.kb_per_split : 0;
    }
    __device__ int kb_end() const
    {
        if constexpr (LAYOUT == kKGrouped)
            return cur_kb1;
        return SPLIT ? min(p.num_kb, kb_begin() + p.kb_per_split) : p.num_kb;
    }
    int cur_kb0 = 0, cur_kb1 = 0;  // K-grouped: the current tile's K blocks

    __device__ bool next(TileCoord &tc, bool report)
    {
        if constexpr (SPLIT) {
            static_assert(LAYOUT == kDense, "the K split is implemented for the dense layout");
            if (next_t++ > 0)
                return false;
            tc.g = 0;
            tc.nb = static_cast<int>(blockIdx.y);
            tc.mb = static_cast<int>(blockIdx.z);
            return true;
        } else if constexpr (LAYOUT == kKGrouped) {
            // tiles group by group, each group's m-blocks fastest
            const int per_group = p.num_mb * p.num_nb;
            const int t = next_t;
            if (t >= p.G * per_group)
                return false;
            next_t += stride;
            tc.g = t / per_group;
            const int within = t - tc.g * per_group;
            tc.nb = within / p.num_mb;
            tc.mb = within - tc.nb * p.num_mb;
            int k0 = __ldg(p.k_offsets + tc.g), k1 = __ldg(p.k_offsets + tc.g + 1);
            if (k0 < 0 || k1 < k0 || k1 > p.K || (k0 % kBK) || (k1 % kBK)) {
                if (report)
                    record_status(kCodeBadGroup, kRoleSched, tc.g);
                k0 = k1 = 0;  // a malformed group is computed as empty
            }
            cur_kb0 = k0 / kBK;
            cur_kb1 = k1 / kBK;
            return true;
        } else if constexpr (LAYOUT == kMasked) {
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
            next_t += stride;
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
                next_t += stride;
                const int per = p.raster * p.num_nb;
                const int grp = t / per;
                const int within = t - grp * per;
                const int rows_here = min(p.raster, p.num_mb - grp * p.raster);
                tc.mb = grp * p.raster + within % rows_here;
                tc.nb = within / rows_here;
                tc.g = 0;
                if constexpr (LAYOUT == kContiguous) {
                    const int g = __ldg(p.m_indices + tc.mb * kBM);
                    if (g < 0) {
                        // padding block: rows stay untouched (flagged if
                        // any of its rows carries a group index)
                        if (report && tc.nb == 0 && padding_block_has_rows(p.m_indices, tc.mb * kBM))
                            record_status(kCodeBadGroup, kRoleSched, 0);
                        continue;
                    }
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

// The spin loop of a wait that did not complete at once.
__device__ __forceinline__ bool wait_bounded_slow(uint32_t bar, uint32_t parity, uint64_t timeout_ns,
                                               volatile int *abort_flag, uint32_t role, uint32_t stage,
                                               bool honour_abort)
{
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

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, uint64_t timeout_ns,
                                             volatile int *abort_flag, uint32_t role,
                                             uint32_t stage, bool honour_abort)
{
    if (mbar_try_wait(bar, parity))
        return true;
    return wait_bounded_slow(bar, parity, timeout_ns, abort_flag, role, stage, honour_abort);
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

// BN: tile width; STAGES: shared-memory ring depth; KS: 128-wide K blocks per
// stage (one 3-D TMA box per operand carries all KS blocks -- the TMA engine
// costs a roughly fixed time per instruction, so bigger boxes move more).
template <int BN_, int STAGES_, int KS_, bool SPLIT_ = false, bool COLSCALE_ = false, int NWG_ = 2,
          bool PROD2_ = false>
struct KernelConfig {
    // PROD2: a second producer warp issues the B boxes while the first
    // issues the A boxes and the scale copies, so the two TMA instructions
    // of a stage are issued in parallel (each holds its issuing thread for
    // a few hundred cycles).
    static constexpr bool PROD2 = PROD2_;
    // COLSCALE: one B scale per column and K block (the K-grouped layout)
    // instead of one per 128x128 block.
    static constexpr bool COLSCALE = COLSCALE_;
    static constexpr int BN = BN_;
    static constexpr int STAGES = STAGES_;
    static constexpr int KS = KS_;
    // SPLIT: the CTAs of a cluster split K; their fp32 partial tiles go
    // through an L2-resident workspace and are summed by the cluster instead
    // of being TMA-stored.
    static constexpr bool SPLIT = SPLIT_;
    // NUM_WG promotion warpgroups split the tile's columns; thread t of each
    // owns tile row t.  Four (the K-split decode tile) halve each thread's
    // columns and double the warps that hide the TMEM-load latency.
    static constexpr int NUM_WG = NWG_;
    static constexpr int BN_WG = BN / NUM_WG;
    // TMEM is read in rounds of at most RMAX columns: a warpgroup whose
    // columns fit beside its accumulator in registers (64, or 40 with four
    // warpgroups and their smaller register budget) pulls its whole partial
    // in one round and frees the buffer before any arithmetic.
    static constexpr int RMAX = BN_WG <= (NUM_WG >= 4 ? 40 : 64) ? BN_WG : 32;
    static constexpr int NUM_PROMO_WARPS = 4 * NUM_WG;
    static constexpr int PRODUCER_WARP = NUM_PROMO_WARPS;
    static constexpr int MMA_WARP = NUM_PROMO_WARPS + 1;
    static constexpr int PRODUCER_B_WARP = NUM_PROMO_WARPS + 2;  // PROD2 only
    static constexpr int THREADS = (NUM_PROMO_WARPS + 2 + (PROD2_ ? 1 : 0)) * 32;
    static constexpr int A_BYTES = kBM * kBK;  // one K block of A
    static constexpr int B_BYTES = BN * kBK;   // one K block of B
    static constexpr int STAGE_BYTES = KS * (A_BYTES + B_BYTES);
    static constexpr int SA_BYTES = KS * kBM * 4;  // LHS scales of a stage
    static constexpr int SB_FLOATS = COLSCALE ? BN : 4;  // B scales per K block
    static constexpr int SB_BYTES = KS * SB_FLOATS * 4;  // (at most 3 weight-block scales, or BN columns)
    // TMEM: NBUF partial buffers of ACC_STRIDE columns (<= 512 in total), so
    // the MMA can run NBUF-1 K blocks ahead of the promotion.
    static constexpr int ACC_STRIDE = (BN + 31) / 32 * 32;
    static constexpr int NBUF = (512 / ACC_STRIDE) < 4 ? (512 / ACC_STRIDE) : 4;
    static constexpr int TMEM_COLS = NBUF * ACC_STRIDE <= 256 ? 256 : 512;
    // + one barrier for the K-split reduction's TMA load
    static constexpr int BAR_BYTES = 8 * (3 * STAGES + 2 * NBUF + 1) + 16;
    // K split: the reduction reads this CTA's rows of all S partials
    // (BN/4 x 128 float4s whatever S is) into the idle operand ring at
    // offset 0, and stages its bf16 rows (at most 64 x BN) after them.
    static constexpr int RED_IN_BYTES = (BN / 4) * kBM * 16;
    static constexpr int RED_OUT_OFFSET = (RED_IN_BYTES + 1023) / 1024 * 1024;
    // Epilogue: each promotion warpgroup stages its 128 rows of the output in
    // shared memory one box at a time and TMA-stores it: boxes of 64 columns
    // (128-byte rows, 128-byte swizzle) and one remainder box.
    static constexpr int EPI_FULL_BOXES = BN_WG / 64;
    static constexpr int EPI_REM = BN_WG % 64;
    static constexpr int EPI_WG_BYTES = kBM * 128;  // 128 rows x 128 bytes
    static constexpr int PIPE_BYTES = STAGES * (STAGE_BYTES + SA_BYTES + SB_BYTES);
    static constexpr int EPI_OFFSET = (PIPE_BYTES + BAR_BYTES + 1023) / 1024 * 1024;
    // One staging buffer per output box when shared memory allows, so a
    // warpgroup stores all its boxes without waiting for an earlier store to
    // finish reading its buffer; else one buffer reused box after box.  A
    // ring too deep for even one buffer per warpgroup (EPI_STAGED false)
    // leaves room only for a small buffer per promotion warp (below).
    static constexpr int EPI_BOXES = EPI_FULL_BOXES + (EPI_REM > 0 ? 1 : 0);
    static constexpr bool EPI_STAGED = 1024 + EPI_OFFSET + NUM_WG * EPI_WG_BYTES <= 232448;
    static constexpr int EPI_BUFS =
        1024 + EPI_OFFSET + NUM_WG * EPI_BOXES * EPI_WG_BYTES <= 232448 ? EPI_BOXES : 1;
    // Without whole-tile staging, each promotion warp stages 32 rows x 32
    // columns of bf16 at a time and writes them back with row-contiguous
    // stores.
    static constexpr int EPI_WARP_BYTES = 32 * 32 * 2;
    static constexpr int SMEM_BYTES =
        1024 /*align slack*/ + EPI_OFFSET +
        (SPLIT ? 0 : EPI_STAGED ? NUM_WG * EPI_BUFS * EPI_WG_BYTES : NUM_PROMO_WARPS * EPI_WARP_BYTES);

    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128: multiple of 16, <= 256");
    static_assert(BN % NUM_WG == 0 && BN_WG % 4 == 0, "promotion columns per warpgroup: a multiple of 4");
    static_assert(BN_WG % 8 == 0 || (SPLIT && !COLSCALE && BN_WG == RMAX),
                  "a column count that is not a multiple of 8 is read in one round and split-reduced");
    static_assert(NUM_WG * 4 + 2 <= 32 && NUM_WG <= 14, "warps per CTA; named barriers 1..NUM_WG, 15 at start-up");
    static_assert(BN_WG <= 128, "a warpgroup's columns must span at most two 128-wide sB blocks");
    static_assert(NBUF >= 2, "double-buffered TMEM at least");
    static_assert(B_BYTES % 1024 == 0, "B tiles must keep 1024-byte swizzle atoms aligned");
    static_assert(KS >= 1 && KS <= 4, "K blocks per stage");
    static_assert(EPI_REM % 8 == 0, "remainder box must be whole 16-byte chunks");
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
    static_assert(SPLIT || EPI_STAGED || BN_WG % 32 == 0, "per-warp epilogue rounds of 32 columns");
    static_assert(!SPLIT || BN_WG % 4 == 0, "split reduction works on float4 columns");
    static_assert(!SPLIT || RED_OUT_OFFSET + 64 * BN * 2 <= STAGES * STAGE_BYTES,
                  "the split reduction's buffers fit in the operand ring");
};

// Loads COLS (multiple of 8, may be 0) consecutive TMEM columns of this
// warp's 32 lanes into r[0..COLS).
// The column offsets are compile-time constants (recursion on Q), so r stays
// in registers.
template <int COLS, int Q = 0>
__device__ __forceinline__ void tmem_load_cols(uint32_t taddr, uint32_t *r)
{
    static_assert(COLS % 4 == 0, "TMEM loads of whole 4-column groups");
    if constexpr (Q + 16 <= COLS) {
        tmem_ld_32x32b_x16(taddr + Q, *reinterpret_cast<uint32_t(*)[16]>(r + Q));
        tmem_load_cols<COLS, Q + 16>(taddr, r);
    } else if constexpr (Q + 8 <= COLS) {
        tmem_ld_32x32b_x8(taddr + Q, *reinterpret_cast<uint32_t(*)[8]>(r + Q));
        tmem_load_cols<COLS, Q + 8>(taddr, r);
    } else if constexpr (Q + 4 <= COLS) {
        tmem_ld_32x32b_x4(taddr + Q, *reinterpret_cast<uint32_t(*)[4]>(r + Q));
        tmem_load_cols<COLS, Q + 4>(taddr, r);
    }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float *v)
{
    __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 h1 = __floats2bfloat162_rn(v[2], v[3]);
    __nv_bfloat162 h2 = __floats2bfloat162_rn(v[4], v[5]);
    __nv_bfloat162 h3 = __floats2bfloat162_rn(v[6], v[7]);
    uint4 u;
    u.x = *reinterpret_cast<uint32_t *>(&h0);
    u.y = *reinterpret_cast<uint32_t *>(&h1);
    u.z = *reinterpret_cast<uint32_t *>(&h2);
    u.w = *reinterpret_cast<uint32_t *>(&h3);
    return u;
}

// ------------------------------------------------------------------ kernel

// A_MN / B_MN: the operand is stored MN-major (A as [K][M], B as [K][N],
// the "t" layouts of the A operand and the "n" layouts of the B operand; dense
// only).  Its stage tile is then loaded as 2-D TMA boxes of 128 M (or N)
// bytes by 128*KS K rows (B: one box per 128 columns, BN % 128 == 0) and
// described to the MMA as an MN-major 128-byte-swizzled operand.
template <int BN, int STAGES, int KS, int LAYOUT, bool SPLIT, bool A_MN = false, bool B_MN = false, int NWG = 2,
          bool PROD2 = false>
__global__ void __launch_bounds__(KernelConfig<BN, STAGES, KS, SPLIT, LAYOUT == kKGrouped, NWG, PROD2>::THREADS, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                    const __grid_constant__ CUtensorMap tmap_b,
                    const __grid_constant__ CUtensorMap tmap_d64,
                    const __grid_constant__ CUtensorMap tmap_drem, const GemmParams p)
{
    using Cfg = KernelConfig<BN, STAGES, KS, SPLIT, LAYOUT == kKGrouped, NWG, PROD2>;
    static_assert(!SPLIT || LAYOUT == kDense, "K split is implemented for the dense layout");
    static_assert(!PROD2 || (!SPLIT && !A_MN && !B_MN && LAYOUT != kKGrouped),
                  "the second producer warp serves K-major persistent tiles");
    static_assert((!A_MN && !B_MN) || LAYOUT == kDense || LAYOUT == kKGrouped,
                  "MN-major operands are implemented for the dense and K-grouped layouts");
    static_assert(LAYOUT != kKGrouped || (A_MN && B_MN), "the K-grouped GEMM is the TN layout");
    static_assert(!B_MN || BN % 128 == 0, "an MN-major B tile is whole 128-column boxes");
    constexpr int BN_WG = Cfg::BN_WG;
    constexpr int RMAX = Cfg::RMAX;
    constexpr int NBUF = Cfg::NBUF;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *a_tiles = smem;                                   // [STAGES*KS][128][128 B]
    uint8_t *b_tiles = smem + STAGES * KS * Cfg::A_BYTES;      // [STAGES*KS][BN][128 B]
    float *sa_tiles = reinterpret_cast<float *>(smem + STAGES * Cfg::STAGE_BYTES);  // [STAGES*KS][128]
    float *sb_tiles = sa_tiles + STAGES * KS * kBM;            // [STAGES*KS][SB_FLOATS]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sb_tiles + STAGES * KS * Cfg::SB_FLOATS);
    uint64_t *full_bar = bars;                 // stage landed (TMA bytes + scale copies)
    uint64_t *empty_bar = bars + STAGES;       // MMAs of the stage done (operand tiles free)
    uint64_t *sread_bar = bars + 2 * STAGES;   // promotion warps have read the stage's scales
    uint64_t *tfull_bar = bars + 3 * STAGES;   // TMEM partial buffer written
    uint64_t *tempty_bar = bars + 3 * STAGES + NBUF;  // TMEM partial buffer read out
    uint64_t *red_bar = bars + 3 * STAGES + 2 * NBUF;  // K split: the reduction's partials landed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(red_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    uint8_t *epi_stage = smem + Cfg::EPI_OFFSET;  // 1024-byte aligned, EPI_BUFS buffers per warpgroup

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    stamp_start(p);

    // Start-up.  The producer warp does not wait for the TMEM allocation:
    // once its lane 0 has initialised the barriers, the warp arrives on the
    // start barrier and begins issuing loads; every other warp waits there
    // until the barriers exist and TMEM is allocated.
    constexpr uint32_t kStartBarrier = 15;
    if (warp == Cfg::PRODUCER_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&tmap_a);
            tma_prefetch_desc(&tmap_b);
            for (int s = 0; s < STAGES; ++s) {
                // full: the elected producer lane's expect-tx arrival plus one
                // cp.async arrival from each of the 32 producer lanes (and
                // the B producer's expect-tx arrival)
                mbar_init(smem_addr(full_bar + s), 1 + 32 + (PROD2 ? 1 : 0));
                mbar_init(smem_addr(empty_bar + s), 1);
                mbar_init(smem_addr(sread_bar + s), Cfg::NUM_PROMO_WARPS);
            }
            for (int b = 0; b < NBUF; ++b) {
                mbar_init(smem_addr(tfull_bar + b), 1);
                mbar_init(smem_addr(tempty_bar + b), Cfg::NUM_PROMO_WARPS);
            }
            mbar_init(smem_addr(red_bar), 1);
            *abort_flag = 0;
            fence_barrier_init();
            // (K split: tmap_d64 describes the partials, tmap_drem the
            // reduction's output rows)
            if (SPLIT || Cfg::EPI_FULL_BOXES > 0)
                tma_prefetch_desc(&tmap_d64);
            if (SPLIT || Cfg::EPI_REM > 0)
                tma_prefetch_desc(&tmap_drem);
        }
        __syncwarp();
        named_barrier_arrive(kStartBarrier, Cfg::THREADS);
    } else {
        if (warp == Cfg::MMA_WARP) {
            tmem_alloc(smem_addr(tmem_slot), Cfg::TMEM_COLS);
            tmem_relinquish_alloc_permit();
        }
        tc_fence_before_sync();
        named_barrier_sync(kStartBarrier, Cfg::THREADS);
        tc_fence_after_sync();
    }
    const uint32_t tmem_base = warp == Cfg::PRODUCER_WARP ? 0u : *tmem_slot;
    const uint64_t tmo = p.timeout_ns;
    // Waits for this CTA's own copies and MMAs in flight before it exits use
    // at least a second, however short the pipeline limit is set.
    const uint64_t drain_tmo = tmo > 1000000000ull ? tmo : 1000000000ull;

    if (warp == Cfg::PRODUCER_WARP) {
        // ------------------------------------------------------ TMA producer
        // The whole warp runs the loop (uniform control flow).  One elected
        // lane issues the two operand boxes of a stage; every lane copies a
        // 16-byte piece of each K block's LHS scales, and lanes 0-2 copy the
        // weight-block scales, all landing on the stage's full barrier.
        TileScheduler<LAYOUT, SPLIT> sched(p);
        TileCoord tc;
        uint32_t stage = 0, phase = 0;
        uint32_t issued = 0;
        // Test hook (dg_set_stall_injection): CTA 0 never fills a stage, so
        // its consumers' waits run out and report DG_ERR_TIMEOUT.
        bool ok = !(p.stall_injection && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0);
        while (ok && sched.next(tc, lane == 0)) {
            const int a_row = (LAYOUT == kMasked ? tc.g * p.M : 0) + tc.mb * kBM;
            // (the K-grouped layout shares one B across its groups)
            const int b_row = (LAYOUT == kKGrouped ? 0 : tc.g * p.N) + tc.nb * BN;
            const int m0 = tc.mb * kBM;
            const float *sa_base = p.sA +
                                   (LAYOUT == kMasked ? static_cast<size_t>(tc.g) * p.num_kb * p.sa_ld : 0) +
                                   m0 + 4 * lane;
            const bool sa_lane_ok = m0 + 4 * lane < p.sa_ld;
            // weight-block scales of the (up to three) 128-row blocks under
            // this tile's columns (lane j copies block nb_first + j, clamped)
            const int nb_first = (tc.nb * BN) / 128;
            const float *sb_src = p.sB + (static_cast<size_t>(tc.g) * p.nbn +
                                          min(nb_first + (lane < 3 ? lane : 0), p.nbn - 1)) * p.num_kb;
            const int kb_end = sched.kb_end();
            for (int kb0 = sched.kb_begin(); kb0 < kb_end; kb0 += KS) {
                if (!warp_wait_bounded(smem_addr(empty_bar + stage), phase ^ 1, tmo, abort_flag,
                                       kRoleProducer, stage) ||
                    !warp_wait_bounded(smem_addr(sread_bar + stage), phase ^ 1, tmo, abort_flag,
                                       kRoleProducer, 64 + stage)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = smem_addr(full_bar + stage);
                if (elect_one()) {
                    mbar_arrive_expect_tx(fb, PROD2 ? KS * Cfg::A_BYTES : Cfg::STAGE_BYTES);
                    if constexpr (A_MN)
                        tma_load_2d(smem_addr(a_tiles + stage * KS * Cfg::A_BYTES), &tmap_a, fb, a_row,
                                    kb0 * kBK);
                    else
                        tma_load_3d(smem_addr(a_tiles + stage * KS * Cfg::A_BYTES), &tmap_a, fb, 0,
                                    a_row, kb0);
                    if constexpr (PROD2) {
                        // (the B producer warp issues the B box)
                    } else if constexpr (B_MN) {
                        // [BN/128 column slices][KS*128 K rows][128 bytes]
#pragma unroll
                        for (int c = 0; c < BN / 128; ++c)
                            tma_load_2d(smem_addr(b_tiles + stage * KS * Cfg::B_BYTES + c * KS * kBK * 128),
                                        &tmap_b, fb, b_row + c * 128, kb0 * kBK);
                    } else {
                        tma_load_3d(smem_addr(b_tiles + stage * KS * Cfg::B_BYTES), &tmap_b, fb, 0,
                                    b_row, kb0);
                    }
                }
#pragma unroll
                for (int q = 0; q < KS; ++q) {
                    const int kb = kb0 + q;
                    const bool in_k = kb < kb_end;
                    const bool sa_ok = in_k && sa_lane_ok;
                    cp_async_16(smem_addr(sa_tiles + (stage * KS + q) * kBM) + 16 * lane,
                                sa_ok ? static_cast<const void *>(sa_base + static_cast<size_t>(kb) * p.sa_ld)
                                      : static_cast<const void *>(p.sA),
                                sa_ok ? 16u : 0u);
                    if constexpr (Cfg::COLSCALE) {
                        // the tile's BN column scales of this K block, in
                        // 16-byte pieces (zeros past N)
#pragma unroll
                        for (int c4 = lane; c4 < BN / 4; c4 += 32) {
                            const int col = tc.nb * BN + 4 * c4;
                            const bool ok_c = in_k && col < p.N;
                            cp_async_16(smem_addr(sb_tiles + (stage * KS + q) * BN) + 16 * c4,
                                        ok_c ? static_cast<const void *>(p.sB + static_cast<size_t>(kb) * p.N + col)
                                             : static_cast<const void *>(p.sB),
                                        ok_c ? 16u : 0u);
                        }
                    } else {
                        if (lane < 3)
                            cp_async_4(smem_addr(sb_tiles + (stage * KS + q) * 4) + 4 * lane,
                                       sb_src + (in_k ? kb : kb_end - 1));
                    }
                }
                cp_async_mbar_arrive_noinc(fb);
                __syncwarp();
                ++issued;
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        // Drain: the last min(STAGES, issued) stages must have landed before
        // the CTA may exit (always true on the normal path).
        if (lane == 0) {
            const uint32_t first = issued > STAGES ? issued - STAGES : 0;
            for (uint32_t i = first; i < issued; ++i)
                wait_bounded(smem_addr(full_bar + i % STAGES), (i / STAGES) & 1, drain_tmo,
                             abort_flag, kRoleDrain, i % STAGES, false);
        }
        __syncwarp();
        if constexpr (SPLIT)
            cluster_sync();  // first cluster barrier of the K-split reduction
    } else if (PROD2 && warp == Cfg::PRODUCER_B_WARP) {
        // ---------------------------------------------------- B box producer
        // The same stages as the A producer, one B box each.  On the normal
        // path the MMA warp waits for every stage, so every box has landed
        // before the CTA exits; after an abort the boxes in flight get a
        // bounded moment to land.
        TileScheduler<LAYOUT, SPLIT> sched(p);
        TileCoord tc;
        uint32_t stage = 0, phase = 0;
        bool ok = !(p.stall_injection && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0);
        while (ok && sched.next(tc, false)) {
            const int b_row = tc.g * p.N + tc.nb * BN;
            const int kb_end = sched.kb_end();
            for (int kb0 = sched.kb_begin(); kb0 < kb_end; kb0 += KS) {
                if (!warp_wait_bounded(smem_addr(empty_bar + stage), phase ^ 1, tmo, abort_flag,
                                       kRoleProducer, 32 + stage)) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    const uint32_t fb = smem_addr(full_bar + stage);
                    mbar_arrive_expect_tx(fb, KS * Cfg::B_BYTES);
                    tma_load_3d(smem_addr(b_tiles + stage * KS * Cfg::B_BYTES), &tmap_b, fb, 0, b_row, kb0);
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        if (!ok && lane == 0) {
            const uint64_t t0 = global_timer_ns();
            while (global_timer_ns() - t0 < 200000ull) {
            }
        }
        __syncwarp();
    } else if (warp == Cfg::MMA_WARP) {
        // ------------------------------------------------------- MMA issuer
        // Uniform loop; the descriptors stay warp-uniform and one elected
        // lane issues the MMAs and the commits.
        TileScheduler<LAYOUT, SPLIT> sched(p);
        TileCoord tc;
        uint32_t stage = 0, phase = 0, acc_i = 0;
        // the most recent commit (barrier, phase parity): it fires once
        // every MMA issued before it has completed
        uint32_t last_bar = 0, last_parity = 0;
        bool ok = true;
        constexpr uint32_t idesc = idesc_e4m3_f32(kBM, BN, A_MN, B_MN);
        // K-major tiles advance 32 bytes per 32-wide K step; MN-major tiles
        // 32 K rows of 128 bytes.  An MN-major B tile's 128-column slices
        // lie KS*128 rows of 128 bytes apart.
        const uint64_t a_desc0 = A_MN ? smem_desc_mn_sw128(smem_addr(a_tiles), KS * kBK * 128)
                                      : smem_desc_k_sw128(smem_addr(a_tiles));
        const uint64_t b_desc0 = B_MN ? smem_desc_mn_sw128(smem_addr(b_tiles), KS * kBK * 128)
                                      : smem_desc_k_sw128(smem_addr(b_tiles));
        constexpr uint64_t a_kstep = A_MN ? (32 * 128) >> 4 : 32 >> 4;
        constexpr uint64_t b_kstep = B_MN ? (32 * 128) >> 4 : 32 >> 4;
        while (ok && sched.next(tc, false)) {
            const int kb_end = sched.kb_end();
            for (int kb0 = sched.kb_begin(); kb0 < kb_end; kb0 += KS) {
                if (!warp_wait_bounded(smem_addr(full_bar + stage), phase, tmo, abort_flag,
                                       kRoleMma, stage)) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int q = 0; q < KS; ++q) {
                    if (kb0 + q >= kb_end)
                        break;
                    const uint32_t buf = acc_i % NBUF, tph = (acc_i / NBUF) & 1;
                    if (!warp_wait_bounded(smem_addr(tempty_bar + buf), tph ^ 1, tmo, abort_flag,
                                           kRoleMma, 16 + buf)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t d_tmem = tmem_base + buf * Cfg::ACC_STRIDE;
                    // descriptor start address advances in 16-byte units
                    const uint64_t ad = a_desc0 + static_cast<uint64_t>(((stage * KS + q) * Cfg::A_BYTES) >> 4);
                    const uint64_t bd =
                        b_desc0 + static_cast<uint64_t>(
                                      (B_MN ? stage * KS * Cfg::B_BYTES + q * kBK * 128 : (stage * KS + q) * Cfg::B_BYTES) >> 4);
                    if (elect_one()) {
#pragma unroll
                        for (int j = 0; j < kBK / 32; ++j)
                            mma_f8f6f4(d_tmem, ad + a_kstep * j, bd + b_kstep * j, idesc, j > 0 ? 1u : 0u);
                        mma_commit(smem_addr(tfull_bar + buf));
                    }
                    __syncwarp();
                    last_bar = smem_addr(tfull_bar + buf);
                    last_parity = tph;
                    ++acc_i;
                }
                if (!ok)
                    break;
                if (elect_one())
                    mma_commit(smem_addr(empty_bar + stage));
                __syncwarp();
                last_bar = smem_addr(empty_bar + stage);
                last_parity = phase;
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        // Drain: every MMA issued by this warp has finished once its most
        // recent commit has fired.
        if (lane == 0 && last_bar != 0)
            wait_bounded(last_bar, last_parity, drain_tmo, abort_flag, kRoleDrain, 32, false);
        __syncwarp();
        if constexpr (SPLIT)
            cluster_sync();  // first cluster barrier of the K-split reduction
    } else {
        // ------------------------------------------------ promotion warps
        const int wg = warp / 4;
        const int quad = warp % 4;
        const int row = quad * 32 + lane;  // tile row == TMEM lane
        const int wg_tid = threadIdx.x % 128;
        const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
        TileScheduler<LAYOUT, SPLIT> sched(p);
        TileCoord tc;
        uint32_t acc_i = 0, stage = 0, phase = 0;
        bool ok = true;
        float acc[BN_WG];

        while (ok && sched.next(tc, false)) {
            const int m_local = tc.mb * kBM + row;  // row index inside the group
            bool row_ok;
            if constexpr (LAYOUT == kDense || LAYOUT == kKGrouped) {
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
            const int col0 = tc.nb * BN + wg * BN_WG;  // first column of this warpgroup
            const int nb_first = (tc.nb * BN) / 128;   // block of sb slot 0
            const int nb_lo = min(col0 / 128, p.nbn - 1);
            const int j_lo = nb_lo - nb_first;
            const int j_hi = min(nb_lo + 1, p.nbn - 1) - nb_first;
            const int boundary = (nb_lo + 1) * 128 - col0;  // local column where sB switches
#pragma unroll
            for (int i = 0; i < BN_WG; ++i)
                acc[i] = 0.0f;

            const int kb_end = sched.kb_end();
            for (int kb0 = sched.kb_begin(); kb0 < kb_end; kb0 += KS) {
                // the stage's scales, then hand the scale slots back
                if (!warp_wait_bounded(smem_addr(full_bar + stage), phase, tmo, abort_flag,
                                       kRolePromote, stage)) {
                    ok = false;
                    break;
                }
                float s_lo[KS], s_hi[KS];
                // column scales (K-grouped): read per element below, so the
                // scale slots are handed back after the stage's K blocks
                const float *sb_cols = sb_tiles + stage * KS * Cfg::SB_FLOATS + wg * BN_WG;
                const uint32_t stage_of_scales = stage;
#pragma unroll
                for (int q = 0; q < KS; ++q) {
                    const float sa = sa_tiles[(stage * KS + q) * kBM + row];
                    if constexpr (Cfg::COLSCALE) {
                        s_lo[q] = s_hi[q] = sa;
                    } else {
                        s_lo[q] = sa * sb_tiles[(stage * KS + q) * 4 + j_lo];
                        s_hi[q] = sa * sb_tiles[(stage * KS + q) * 4 + j_hi];
                    }
                }
                if constexpr (!Cfg::COLSCALE) {
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(smem_addr(sread_bar + stage));
                }
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
#pragma unroll
                for (int q = 0; q < KS; ++q) {
                    if (kb0 + q >= kb_end)
                        break;
                    const uint32_t buf = acc_i % NBUF, tph = (acc_i / NBUF) & 1;
                    if (!warp_wait_bounded(smem_addr(tfull_bar + buf), tph, tmo, abort_flag,
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
                            // every column of this buffer is in registers: free it
                            tc_fence_before_sync();
                            __syncwarp();
                            if (lane == 0)
                                mbar_arrive(smem_addr(tempty_bar + buf));
                        }
                        if constexpr (BN_WG % 8 != 0) {
                            // columns in groups of 4 (one round, per-block
                            // scales): a warpgroup starting at 4 mod 8 can
                            // meet the 128-column scale boundary inside an
                            // 8-column group
#pragma unroll
                            for (int g4 = 0; g4 < RMAX; g4 += 4) {
                                const float sc = (c0 + g4 >= boundary) ? s_hi[q] : s_lo[q];
#pragma unroll
                                for (int i = 0; i < 4; ++i)
                                    acc[c0 + g4 + i] = fmaf(__uint_as_float(r[g4 + i]), sc, acc[c0 + g4 + i]);
                            }
                            continue;
                        }
#pragma unroll
                        for (int g8 = 0; g8 < RMAX; g8 += 8) {
                            if (whole || g8 < TAIL) {
                                if constexpr (Cfg::COLSCALE) {
                                    // sA[kb,m] * sB[kb,n] per column (a
                                    // broadcast shared-memory read)
                                    const float *sbq = sb_cols + q * Cfg::SB_FLOATS + c0 + g8;
#pragma unroll
                                    for (int i = 0; i < 8; ++i)
                                        acc[c0 + g8 + i] = fmaf(__uint_as_float(r[g8 + i]), s_lo[q] * sbq[i],
                                                                acc[c0 + g8 + i]);
                                } else {
                                    const float sc = (c0 + g8 >= boundary) ? s_hi[q] : s_lo[q];
#pragma unroll
                                    for (int i = 0; i < 8; ++i)
                                        acc[c0 + g8 + i] = fmaf(__uint_as_float(r[g8 + i]), sc, acc[c0 + g8 + i]);
                                }
                            }
                        }
                    }
                    ++acc_i;
                }
                if constexpr (Cfg::COLSCALE) {
                    if (ok) {
                        __syncwarp();
                        if (lane == 0)
                            mbar_arrive(smem_addr(sread_bar + stage_of_scales));
                    }
                }
                if (!ok)
                    break;
            }

            // ------------------------------------------------------ epilogue
            if constexpr (SPLIT) {
                // K split: this split's fp32 partial tile goes to the
                // workspace as [column quad][row] float4s, so the 32 rows of
                // a warp write 512 contiguous bytes per store.  A warp that
                // gave up on a wait writes NaN instead: the cluster's sums
                // for its columns then show the failure rather than add a
                // stale partial left in the workspace by an earlier call.
                const size_t tile = static_cast<size_t>(tc.mb) * p.num_nb + tc.nb;
                float4 *dst = reinterpret_cast<float4 *>(p.ws) +
                              ((tile * p.ksplit + cluster_ctarank()) * (BN / 4) + wg * (BN_WG / 4)) * kBM + row;
                const float nan = __int_as_float(0x7FC00000);
#pragma unroll
                for (int c = 0; c < BN_WG; c += 4)
                    dst[(c / 4) * kBM] = ok ? make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3])
                                            : make_float4(nan, nan, nan, nan);
                continue;
            }
            // A warpgroup stores its 128 rows with whole-tile TMA boxes when
            // every row may be written: dense rows past M are clipped by the
            // tensor extent, while grouped layouts must not touch rows outside
            // the group, so a warpgroup with any such row stores row by row.
            // A warp that gave up on a wait still joins the first barrier
            // below; if any warp of the warpgroup gave up, the whole
            // warpgroup leaves together, so no warp can be left waiting at
            // a later named barrier for warps that are gone.
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
            if constexpr (LAYOUT == kKGrouped) {
                // fp32 D_g, row by row
                if (row_ok)
                    store_row_f32<BN_WG>(p.D32 + (static_cast<size_t>(tc.g) * p.M + m_local) * p.N + col0, acc,
                                         col0, p.N);
                continue;
            }
            const bool tile_rows_ok = Cfg::EPI_STAGED && named_barrier_and(
                1 + wg, 128, LAYOUT == kDense ? (tc.mb * kBM < p.M) : row_ok);
            if (tile_rows_ok) {
                const int grow0 = (LAYOUT == kMasked ? tc.g * p.M : 0) + tc.mb * kBM;
#pragma unroll
                for (int bx = 0; bx < Cfg::EPI_BOXES; ++bx) {
                    const bool full = bx < Cfg::EPI_FULL_BOXES;
                    const int cbase = bx * 64;
                    const int ncols = full ? 64 : Cfg::EPI_REM;
                    if (col0 + cbase >= p.N)
                        break;  // this box (and any after it) lies past N
                    const uint32_t stg =
                        smem_addr(epi_stage + (wg * Cfg::EPI_BUFS + bx % Cfg::EPI_BUFS) * Cfg::EPI_WG_BYTES);
                    // the store that last used this staging buffer (one per
                    // box, the most recent EPI_BUFS - 1 may still be pending)
                    // must have finished reading it before it is overwritten
                    if (wg_tid == 0)
                        bulk_wait_group_read<Cfg::EPI_BUFS - 1>();
                    named_barrier_sync(1 + wg, 128);
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        if (ch * 8 < ncols) {
                            // full boxes: 128-byte rows, 16-byte chunk index
                            // XOR (row % 8); remainder: dense rows of ncols*2
                            const uint32_t off =
                                full ? static_cast<uint32_t>(row * 128 + ((ch ^ (row & 7)) * 16))
                                     : static_cast<uint32_t>(row * ncols * 2 + ch * 16);
                            st_shared_v4(stg + off, pack_bf16x8(acc + cbase + ch * 8));
                        }
                    }
                    fence_proxy_async_smem();
                    named_barrier_sync(1 + wg, 128);
                    if (wg_tid == 0) {
                        tma_store_2d(full ? static_cast<const void *>(&tmap_d64)
                                          : static_cast<const void *>(&tmap_drem),
                                     stg, col0 + cbase, grow0);
                        bulk_commit_group();
                    }
                }
            } else if constexpr (Cfg::EPI_STAGED) {
                if (row_ok) {
                    const size_t grow = (LAYOUT == kMasked ? static_cast<size_t>(tc.g) * p.M : 0) +
                                        static_cast<size_t>(m_local);
                    __nv_bfloat16 *drow = p.D + grow * p.N + col0;
#pragma unroll
                    for (int c = 0; c < BN_WG; c += 8)
                        if (col0 + c < p.N)
                            *reinterpret_cast<uint4 *>(drow + c) = pack_bf16x8(acc + c);
                }
            } else {
                // Each warp puts 32 rows x 32 columns of bf16 into its own
                // 2 KB buffer (16-byte chunk c of row r at slot c ^ ((r/2) % 4):
                // conflict-free both ways) and reads them back so that four
                // lanes cover one row's 64 bytes: every store instruction
                // writes 8 row segments.  Rows that may not be written are
                // skipped by the lanes that hold them.
                const uint32_t wbuf = smem_addr(epi_stage) + static_cast<uint32_t>(warp * Cfg::EPI_WARP_BYTES);
                const unsigned rows = __ballot_sync(0xFFFFFFFFu, row_ok);
                const size_t grow0 = (LAYOUT == kMasked ? static_cast<size_t>(tc.g) * p.M : 0) +
                                     static_cast<size_t>(tc.mb) * kBM + static_cast<size_t>(quad * 32);
#pragma unroll
                for (int cb = 0; cb < BN_WG; cb += 32) {
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch)
                        st_shared_v4(wbuf + lane * 64 + ((ch ^ ((lane >> 1) & 3)) * 16),
                                     pack_bf16x8(acc + cb + ch * 8));
                    __syncwarp();
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int r = 8 * j + lane / 4;
                        const int ch = lane % 4;
                        const uint4 v = ld_shared_v4u(wbuf + r * 64 + ((ch ^ ((r >> 1) & 3)) * 16));
                        const int gcol = col0 + cb + ch * 8;
                        if (((rows >> r) & 1u) != 0u && gcol < p.N)
                            *reinterpret_cast<uint4 *>(p.D + (grow0 + r) * p.N + gcol) = v;
                    }
                    __syncwarp();
                }
            }
        }
        if constexpr (SPLIT) {
            __threadfence();
            cluster_sync();  // every split's partial tile is in the workspace
        }
        // all output stores of this warpgroup complete before the CTA exits
        if (wg_tid == 0)
            bulk_wait_group<0>();
        __syncwarp();
    }

    __syncthreads();
    if constexpr (SPLIT) {
        // K-split reduction: CTA `rank` owns rows [rank*128/S, (rank+1)*128/S)
        // of the tile and sums the S partials of those rows from the
        // workspace in split order (a fixed order, so results do not depend
        // on timing), then rounds to bf16.
        const int S = p.ksplit;
        const uint32_t rank = cluster_ctarank();
        TileScheduler<LAYOUT, SPLIT> sched(p);
        TileCoord tc;
        if (sched.next(tc, false)) {
            // rows [r0, r1) of the tile: S need not divide 128
            const int r0 = static_cast<int>(rank) * kBM / S;
            const int rows_per = (static_cast<int>(rank) + 1) * kBM / S - r0;
            constexpr int C4 = BN / 4;
            const size_t tile = static_cast<size_t>(tc.mb) * p.num_nb + tc.nb;
            const float4 *src0 = reinterpret_cast<const float4 *>(p.ws) + tile * S * C4 * kBM;
            if (p.D32 == nullptr && S >= 2 && kBM % S == 0) {
                // (the same condition under which the host built the two maps)
                // bf16 output.  One TMA box brings this CTA's rows of all S
                // partials, [S][C4][rows_per] float4s, into the idle operand
                // ring; the sums (in split order, as below) are rounded,
                // staged as [rows_per][BN] bf16 and stored with one TMA box
                // (rows past M and columns past N are clipped).
                const float4 *red_in = reinterpret_cast<const float4 *>(smem);
                uint8_t *red_out = smem + Cfg::RED_OUT_OFFSET;
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
                const int r = r0 + lr;
                // all S loads in flight at once (S <= 16), then the sum in
                // split order
                float4 v[16];
#pragma unroll
                for (int src = 0; src < 16; ++src)
                    if (src < S)
                        v[src] = __ldcg(src0 + (static_cast<size_t>(src) * C4 + c4) * kBM + r);
                float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int src = 0; src < 16; ++src) {
                    if (src < S) {
                        sum.x += v[src].x;
                        sum.y += v[src].y;
                        sum.z += v[src].z;
                        sum.w += v[src].w;
                    }
                }
                const int grow = tc.mb * kBM + r;
                const int gcol = tc.nb * BN + c4 * 4;
                if (grow < p.M && gcol < p.N && p.D32) {
                    // accumulate form: fp32 C + sum
                    const size_t off = static_cast<size_t>(grow) * p.N + gcol;
                    const float4 cv = *reinterpret_cast<const float4 *>(p.C + off);
                    *reinterpret_cast<float4 *>(p.D32 + off) =
                        make_float4(cv.x + sum.x, cv.y + sum.y, cv.z + sum.z, cv.w + sum.w);
                } else if (grow < p.M && gcol < p.N) {
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
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace dg
