// dg_api.cu -- host side of the C ABI declared in include/dg_b200.h:
// argument validation, tile-shape choice, TMA descriptor encoding and kernel
// launch.  All arithmetic of the GEMM runs in fp8_gemm_kernel.cuh (one CTA
// per tile), fp8_gemm_pair_kernel.cuh (a CTA pair per 256-row tile) and
// fp8_gemm_bs_kernel.cuh (the UE8M0 block-scaled mode and its scale packing).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/dg_b200.h"
#include "fp8_gemm_bs_kernel.cuh"
#include "fp8_gemm_kernel.cuh"
#include "fp8_gemm_pair_kernel.cuh"

namespace {

using dg::GemmParams;
using dg::KernelConfig;
using dg::PairConfig;

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;

std::atomic<int> g_num_sms_cap{0};
std::atomic<uint64_t> g_timeout_ns{kDefaultTimeoutNs};
std::atomic<int> g_stall_injection{0};
std::atomic<unsigned long long *> g_stamps{nullptr};  // dg_set_timing_stamps
int g_sm_count[kMaxDevices] = {0};

// ------------------------------------------------------------ driver entry

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// Tensor maps are cached per (base pointer, data type, shape, strides, box,
// swizzle, L2 promotion): a call repeated on the same buffers encodes none,
// which keeps the host cost of small, frequent calls (decode steps) down.
// The cache is a small set-associative
// table under a mutex; a miss encodes with cuTensorMapEncodeTiled and
// replaces the set's entries in turn.  The device a map is used on does not
// enter the key: the encoded map holds only the address and the layout.
struct TmapKey {
    const void *base;
    uint64_t dims[4];
    uint64_t strides[3];
    uint32_t box[4];
    uint32_t rank, dtype, swizzle, promo;
    bool operator==(const TmapKey &o) const { return std::memcmp(this, &o, sizeof(*this)) == 0; }
};

constexpr int kTmapSets = 64;
constexpr int kTmapWays = 4;
struct TmapEntry {
    bool valid = false;
    TmapKey key;
    CUtensorMap map;
};
std::mutex g_tmap_mutex;
TmapEntry g_tmap_cache[kTmapSets][kTmapWays];
int g_tmap_next_way[kTmapSets] = {};
std::atomic<uint64_t> g_tmap_encodes{0};  // encodes performed (cache misses)

bool encode_cached(CUtensorMap *map, CUtensorMapDataType dtype, uint32_t rank, const void *base,
                   const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box,
                   CUtensorMapSwizzle swizzle, CUtensorMapL2promotion promo)
{
    TmapKey k;
    std::memset(&k, 0, sizeof(k));  // padding bytes take part in the comparison
    k.base = base;
    for (uint32_t i = 0; i < rank; ++i) {
        k.dims[i] = dims[i];
        k.box[i] = box[i];
        if (i + 1 < rank)
            k.strides[i] = strides[i];
    }
    k.rank = rank;
    k.dtype = static_cast<uint32_t>(dtype);
    k.swizzle = static_cast<uint32_t>(swizzle);
    k.promo = static_cast<uint32_t>(promo);
    uint64_t h = reinterpret_cast<uintptr_t>(base) >> 4;
    for (uint32_t i = 0; i < rank; ++i)
        h = h * 1000003u ^ (k.dims[i] * 31u + k.box[i]);
    h = h * 1000003u ^ (k.dtype * 7u + k.swizzle * 3u + k.promo);
    const int set = static_cast<int>((h ^ (h >> 29)) % kTmapSets);
    std::lock_guard<std::mutex> lock(g_tmap_mutex);
    for (TmapEntry &e : g_tmap_cache[set]) {
        if (e.valid && e.key == k) {
            *map = e.map;
            return true;
        }
    }
    EncodeTiledFn enc = encode_fn();
    if (!enc)
        return false;
    cuuint32_t estr[4] = {1, 1, 1, 1};
    if (enc(map, dtype, rank, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    g_tmap_encodes.fetch_add(1);
    TmapEntry &slot = g_tmap_cache[set][g_tmap_next_way[set]];
    g_tmap_next_way[set] = (g_tmap_next_way[set] + 1) % kTmapWays;
    slot.valid = true;
    slot.key = k;
    slot.map = *map;
    return true;
}

// An e4m3 operand [rows][K] viewed in 3-D as (byte within a 128-wide K
// block, row, K block), so that one box of [ks][box_rows][128 bytes] fetches
// ks consecutive K blocks of box_rows rows, each block a 128-byte-swizzled
// K-major tile.
bool make_tmap_operand(CUtensorMap *map, const void *base, uint64_t K, uint64_t rows,
                       uint32_t box_rows, uint32_t ks)
{
    cuuint64_t dims[3] = {128, rows, K / 128};
    cuuint64_t strides[2] = {K, 128};
    cuuint32_t box[3] = {128, box_rows, ks};
    return encode_cached(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

// An MN-major e4m3 operand stored [K][inner] (inner = M for A, N for B):
// 2-D boxes of 128 inner bytes by box_k K rows, 128-byte swizzled.
bool make_tmap_mn(CUtensorMap *map, const void *base, uint64_t inner, uint64_t K, uint32_t box_k)
{
    cuuint64_t dims[2] = {inner, K};
    cuuint64_t strides[1] = {inner};
    cuuint32_t box[2] = {128, box_k};
    return encode_cached(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

// 2-D bf16 matrix [rows][inner] (the output), box [box_rows][box_inner].
bool make_tmap_bf16(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows,
                    uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swizzle)
{
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {box_inner, box_rows};
    return encode_cached(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, swizzle,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE);
}

// The K-split workspace [tiles][S][BN/4][128] float4s viewed in 4-D as
// (float within a column quad's 128 rows, column quad, split, tile), with a
// box of one CTA's rows_per rows of every column quad and split of one tile.
bool make_tmap_split_ws(CUtensorMap *map, const float *ws, int bn, int S, uint64_t tiles, int rows_per)
{
    const uint64_t c4 = static_cast<uint64_t>(bn / 4);
    cuuint64_t dims[4] = {4ull * 128ull, c4, static_cast<uint64_t>(S), tiles};
    cuuint64_t strides[3] = {4ull * 128ull * 4ull, 4ull * 128ull * 4ull * c4,
                             4ull * 128ull * 4ull * c4 * static_cast<uint64_t>(S)};
    cuuint32_t box[4] = {static_cast<cuuint32_t>(4 * rows_per), static_cast<cuuint32_t>(c4),
                         static_cast<cuuint32_t>(S), 1};
    return encode_cached(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, ws, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

// ------------------------------------------------------------------- device

int current_device()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return -1;
    return dev;
}

int device_sm_count(int dev)
{
    if (dev < 0 || dev >= kMaxDevices)
        return 0;
    if (g_sm_count[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return 0;
        g_sm_count[dev] = n;
    }
    return g_sm_count[dev];
}

int effective_sms(int dev)
{
    const int hw = device_sm_count(dev);
    const int cap = g_num_sms_cap.load();
    return (cap > 0 && cap < hw) ? cap : hw;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Per-device fp32 workspace of the K-split path, allocated on first use and
// grown when a larger one is needed; kept until process exit.
std::mutex g_ws_mutex;
void *g_ws_ptr[kMaxDevices] = {};
size_t g_ws_bytes[kMaxDevices] = {};
std::atomic<uint64_t> g_device_allocs{0};  // cudaMalloc calls made (dg_get_device_allocations)

dg_status_t split_workspace(int dev, size_t bytes, void **out)
{
    if (dev < 0 || dev >= kMaxDevices)
        return DG_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_ws_mutex);
    if (g_ws_bytes[dev] < bytes) {
        if (g_ws_ptr[dev]) {
            if (cudaFree(g_ws_ptr[dev]) != cudaSuccess)
                return DG_ERR_CUDA;
            g_ws_ptr[dev] = nullptr;
            g_ws_bytes[dev] = 0;
        }
        void *ptr = nullptr;
        g_device_allocs.fetch_add(1);
        if (cudaMalloc(&ptr, bytes) != cudaSuccess) {
            (void)cudaGetLastError();
            return DG_ERR_CUDA;
        }
        g_ws_ptr[dev] = ptr;
        g_ws_bytes[dev] = bytes;
    }
    *out = g_ws_ptr[dev];
    return DG_OK;
}

// ---------------------------------------------------------- configurations

// The tile widths compiled into the library.  Each has a pipeline depth that
// fills the 227 KB of shared memory (one CTA per SM).  128x256 comes twice:
// three stages with whole-tile staged TMA stores (cheaper per tile: short K
// ranges) and four stages with per-warp stores (cheaper per K block: long K
// ranges); the cost model picks between them.
struct TileChoice {
    int bn;
    int stages;
    int ks;      // 128-wide K blocks per pipeline stage
    int split;   // 0: persistent tiles; 1: K split over a cluster (dense only)
    double kb_ns;    // measured time of one K block of one tile (cost model, us)
    int pair;        // 1: 256 x bn tiles on CTA pairs (cta_group::2)
    double tile_us;  // per-tile fill, drain and epilogue (cost model, us)
    int wg = 2;      // promotion warpgroups
    int rebal = 0;   // pair tiles: registers rebalanced with setmaxnreg (always for wg >= 3)
    int masked_only = 0;  // taken only by the masked layout's decode-sized groups
    int nmajor_split = 0;  // the K split of an N-major B (whole 128-column boxes) only
};
constexpr TileChoice kTileChoices[] = {
    {112, 3, 2, 0, 0.41, 0, 1.9}, {128, 5, 1, 0, 0.53, 0, 1.9}, {224, 2, 2, 0, 0.78, 0, 1.9},
    {256, 3, 1, 0, 0.68, 0, 1.9}, {144, 3, 2, 1, 0.40, 0, 1.9, 3}, {160, 3, 2, 0, 0.441, 1, 2.2},
    {192, 3, 2, 0, 0.50, 1, 2.2, 3}, {128, 3, 2, 0, 0.50, 0, 1.9, 2, 0, 1}, {128, 3, 2, 1, 0.40, 0, 1.9, 2, 0, 0, 1},
    {256, 4, 1, 0, 0.655, 0, 2.6},
};
// The masked layout's tile for decode-sized groups (at most two 128-row
// blocks per group): HBM-bound on the weights, it keeps six K blocks in
// flight per SM in three stages of two-K-block boxes (half the TMA
// instructions of one-K-block stages), issued by two producer warps (A and
// scales, B) in parallel, and stores rows directly.
constexpr int kMaskedDecodeTile = 7;
constexpr int kSplitFixedNs = 1500;  // cluster reduction + pipeline fill of a split CTA

// Tile width pinned by dg_set_block_n (0 = the cost model decides); its
// initial value comes from DG_FORCE_BLOCK_N=<n>.
std::atomic<int> g_forced_bn{-1};

int forced_block_n()
{
    int v = g_forced_bn.load();
    if (v < 0) {
        const char *e = std::getenv("DG_FORCE_BLOCK_N");
        g_forced_bn.compare_exchange_strong(v, e ? std::atoi(e) : 0);
        v = g_forced_bn.load();
    }
    return v;
}

// Tile family restriction (dg_set_tile_family): -1 none, 0 one-CTA tiles
// only, 1 pair tiles only.  Its initial value comes from DG_FORCE_PAIR=0|1.
std::atomic<int> g_forced_pair{-2};

int forced_pair()
{
    int v = g_forced_pair.load();
    if (v == -2) {
        const char *e = std::getenv("DG_FORCE_PAIR");
        const int init = (e && e[0]) ? (std::atoi(e) != 0 ? 1 : 0) : -1;
        g_forced_pair.compare_exchange_strong(v, init);
        v = g_forced_pair.load();
    }
    return v;
}

// DG_PRINT_CONFIGS=1 prints each call's plan to stderr.
bool print_configs()
{
    static int v = -1;
    if (v < 0) {
        const char *e = std::getenv("DG_PRINT_CONFIGS");
        v = (e && e[0] && e[0] != '0') ? 1 : 0;
    }
    return v == 1;
}

struct Plan {
    TileChoice c;
    int ksplit;  // CTAs per cluster sharing a tile's K range (1 = none)
};

int max_active_clusters(const TileChoice &c, int S);

// Deterministic choice, no autotuning (lqnn.cn article, section
// "完全JIT设计"; non-power-of-two BLOCK_N to fill the SMs, section
// "非对齐块大小"): waves of tiles over the SMs times the time of one tile.
// When a problem has too few tiles to fill the GPU (decode shapes), the K
// range of each tile may be split over a cluster of 2..16 CTAs.  Pair tiles
// (256 rows on two SMs) are taken only by problems with at least one full
// wave of them.  m_blocks counts 128-row blocks, pair_rows 256-row ones.
// Operand layouts restrict the choice: MN-major operands run on one-CTA
// tiles only (kNoPair), and an MN-major B needs whole 128-column boxes
// (kWholeBoxes: BN % 128 == 0, no K split).
constexpr int kNoPair = 1;
constexpr int kWholeBoxes = 2;

Plan choose_plan(int64_t m_blocks, int64_t pair_rows, int N, int num_kb, int sms, bool allow_split,
                 int limits = 0)
{
    Plan best{kTileChoices[0], 1};
    double best_cost = 1e300;
    if (limits & kWholeBoxes) {
        // (an N-major B splits K only on the 128-column split tile)
        for (const TileChoice &c : kTileChoices)
            if (!c.pair && !c.split && c.bn % 128 == 0) {
                best = Plan{c, 1};
                break;
            }
    }
    for (const TileChoice &c : kTileChoices) {
        const bool forced = forced_block_n() > 0;
        if (forced && c.bn != forced_block_n())
            continue;
        if ((limits & (kNoPair | kWholeBoxes)) && c.pair)
            continue;
        if ((limits & kWholeBoxes) && c.bn % 128 != 0)
            continue;
        if (forced_pair() >= 0 && c.pair != forced_pair())
            continue;
        if (c.masked_only)
            continue;
        if (c.nmajor_split != ((limits & kWholeBoxes) != 0 && c.split))
            continue;
        if (c.pair) {
            const int pairs = sms / 2;
            const int64_t tiles = pair_rows * ((N + c.bn - 1) / c.bn);
            if (pairs <= 0 || (tiles < pairs && forced_pair() != 1))
                continue;
            const int64_t waves = (tiles + pairs - 1) / pairs;
            const double cost = static_cast<double>(waves) * (num_kb * c.kb_ns + c.tile_us);
            if (cost < best_cost) {
                best_cost = cost;
                best = Plan{c, 1};
            }
            continue;
        }
        const int64_t tiles = m_blocks * ((N + c.bn - 1) / c.bn);
        if (!c.split) {
            const int64_t waves = (tiles + sms - 1) / sms;
            const double cost = static_cast<double>(waves) * (num_kb * c.kb_ns + c.tile_us);
            if (cost < best_cost) {
                best_cost = cost;
                best = Plan{c, 1};
            }
            continue;
        }
        if (!allow_split)
            continue;
        for (int S = 2; S <= 16; S *= 2) {
            const int kbps = (num_kb + S - 1) / S;
            if (kbps < 2)
                break;
            const int S_eff = (num_kb + kbps - 1) / kbps;
            if (S_eff != S)
                continue;
            if (tiles > max_active_clusters(c, S))
                continue;
            const double cost = kbps * c.kb_ns + c.tile_us + kSplitFixedNs * 1e-3;
            if (cost < best_cost) {
                best_cost = cost;
                best = Plan{c, S};
            }
        }
    }
    return best;
}

// Rasterisation: tiles are visited in groups of `raster` m-block rows (pair
// rows for pair tiles), column by column inside a group, so the CTAs working
// at one time share the group's rows of A and walk B column by column.  The
// group height is chosen so that the group's A rows (rows_per_block x K
// bytes each) take at most about a third of L2 (40 MB): they then stay
// resident while B streams past, and A is read from DRAM about once per
// group instead of once per wave of tiles (at most 16 blocks per group).
// DG_RASTER=<n> overrides the group height (read once; for tuning sweeps).
int choose_raster(int num_mb, int rows_per_block, int K)
{
    static int forced = -1;
    if (forced < 0) {
        const char *e = std::getenv("DG_RASTER");
        forced = e ? std::atoi(e) : 0;
    }
    constexpr double kBandBytes = 40.0 * 1024 * 1024;
    const double block_bytes = static_cast<double>(rows_per_block) * (K > 0 ? K : 1);
    int want = forced > 0 ? forced : static_cast<int>(kBandBytes / block_bytes);
    want = want < 1 ? 1 : (want > 16 && forced <= 0 ? 16 : want);
    return num_mb < want ? (num_mb > 0 ? num_mb : 1) : want;
}

template <int BN, int STAGES, int KS, int LAYOUT, bool SPLIT, bool A_MN = false, bool B_MN = false, int NWG = 2,
          bool PROD2 = false>
dg_status_t launch_kernel(const void *A, uint64_t a_rows, const void *B, uint64_t b_rows,
                          const GemmParams &p, int grid, cudaStream_t stream)
{
    using Cfg = KernelConfig<BN, STAGES, KS, SPLIT, LAYOUT == dg::kKGrouped, NWG, PROD2>;
    CUtensorMap ta, tb;
    const bool ok_a = A_MN ? make_tmap_mn(&ta, A, a_rows, static_cast<uint64_t>(p.K), KS * dg::kBK)
                           : make_tmap_operand(&ta, A, static_cast<uint64_t>(p.K), a_rows, dg::kBM, KS);
    const bool ok_b = B_MN ? make_tmap_mn(&tb, B, b_rows, static_cast<uint64_t>(p.K), KS * dg::kBK)
                           : make_tmap_operand(&tb, B, static_cast<uint64_t>(p.K), b_rows, BN, KS);
    if (!ok_a || !ok_b)
        return DG_ERR_CUDA;
    const uint64_t d_rows = a_rows;
    // output boxes of 32 rows: 64 columns with 128-byte swizzle, and the
    // warpgroup's remainder columns unswizzled
    CUtensorMap td64, tdrem;
    if (!make_tmap_bf16(&td64, p.D, static_cast<uint64_t>(p.N), d_rows, 64, dg::kBM,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return DG_ERR_CUDA;
    if (Cfg::EPI_REM > 0) {
        if (!make_tmap_bf16(&tdrem, p.D, static_cast<uint64_t>(p.N), d_rows, Cfg::EPI_REM, dg::kBM,
                            CU_TENSOR_MAP_SWIZZLE_NONE))
            return DG_ERR_CUDA;
    } else {
        tdrem = td64;
    }
    if (SPLIT && p.D != nullptr && p.ksplit >= 2 && dg::kBM % p.ksplit == 0) {
        // the K-split reduction's maps: the partials (in place of the
        // epilogue's 64-column boxes) and one CTA's output rows
        const int rows_per = dg::kBM / p.ksplit;
        const uint64_t tiles = static_cast<uint64_t>(p.num_mb) * static_cast<uint64_t>(p.num_nb);
        if (!make_tmap_split_ws(&td64, p.ws, BN, p.ksplit, tiles, rows_per) ||
            !make_tmap_bf16(&tdrem, p.D, static_cast<uint64_t>(p.N), d_rows, BN, rows_per,
                            CU_TENSOR_MAP_SWIZZLE_NONE))
            return DG_ERR_CUDA;
    }
    auto kern = dg::fp8_gemm_kernel<BN, STAGES, KS, LAYOUT, SPLIT, A_MN, B_MN, NWG, PROD2>;
    static std::atomic<bool> attr_set[kMaxDevices];
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices)
        return DG_ERR_CUDA;
    if (!attr_set[dev].load()) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg::SMEM_BYTES) != cudaSuccess)
            return DG_ERR_CUDA;
        if (SPLIT && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                         cudaSuccess)
            return DG_ERR_CUDA;
        attr_set[dev].store(true);
    }
    if (SPLIT) {
        // 3-D grid: x the K split (a cluster along x), y the column tile, z
        // the 128-row block -- one tile per cluster
        (void)grid;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(p.ksplit), static_cast<unsigned>(p.num_nb),
                           static_cast<unsigned>(p.num_mb));
        cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
        cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(p.ksplit);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kern, ta, tb, td64, tdrem, p) != cudaSuccess) {
            (void)cudaGetLastError();
            return DG_ERR_CUDA;
        }
        return DG_OK;
    }
    kern<<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(ta, tb, td64, tdrem, p);
    if (cudaPeekAtLastError() != cudaSuccess) {
        (void)cudaGetLastError();
        return DG_ERR_CUDA;
    }
    return DG_OK;
}

// Pair tiles: a cluster of two CTAs per 256 x BN tile, persistent over
// tiles; grid = 2 x (pairs in use).
template <int BN, int STAGES, int KS, int LAYOUT, int NWG, bool REBAL = false>
dg_status_t launch_pair(const void *A, uint64_t a_rows, const void *B, uint64_t b_rows,
                        const GemmParams &p, int grid, cudaStream_t stream)
{
    using Cfg = PairConfig<BN, STAGES, KS, NWG, REBAL>;
    CUtensorMap ta, tb;
    if (!make_tmap_operand(&ta, A, static_cast<uint64_t>(p.K), a_rows, dg::kBM, KS) ||
        !make_tmap_operand(&tb, B, static_cast<uint64_t>(p.K), b_rows, Cfg::BN_HALF, KS))
        return DG_ERR_CUDA;
    // output boxes of 128 rows: 32 columns with 64-byte swizzle, and a
    // unswizzled remainder box of the leftover columns
    CUtensorMap tdbox, tdrem;
    if (!make_tmap_bf16(&tdbox, p.D, static_cast<uint64_t>(p.N), a_rows, Cfg::EPI_BOX, dg::kBM,
                        CU_TENSOR_MAP_SWIZZLE_64B))
        return DG_ERR_CUDA;
    if (Cfg::EPI_REM > 0) {
        if (!make_tmap_bf16(&tdrem, p.D, static_cast<uint64_t>(p.N), a_rows, Cfg::EPI_REM, dg::kBM,
                            CU_TENSOR_MAP_SWIZZLE_NONE))
            return DG_ERR_CUDA;
    } else {
        tdrem = tdbox;
    }
    auto kern = dg::fp8_gemm_pair_kernel<BN, STAGES, KS, LAYOUT, NWG, REBAL>;
    static std::atomic<bool> attr_set[kMaxDevices];
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices)
        return DG_ERR_CUDA;
    if (!attr_set[dev].load()) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg::SMEM_BYTES) != cudaSuccess)
            return DG_ERR_CUDA;
        if (Cfg::REBALANCE) {
            // setmaxnreg moves registers between warpgroups inside the
            // block's launch allocation; if the compiled kernel were launched
            // with fewer registers than the budgets add up to, the increase
            // would wait forever, so such a build is refused here.
            cudaFuncAttributes fa{};
            if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess)
                return DG_ERR_CUDA;
            if (fa.numRegs < Cfg::LAUNCH_REGS)
                return DG_ERR_UNSUPPORTED;
        }
        attr_set[dev].store(true);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (print_configs()) {
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
            (void)cudaGetLastError();
            n = -1;
        }
        std::fprintf(stderr, "[dg] pair kernel: grid %d CTAs, %d co-resident pairs possible, smem %d B\n",
                     grid, n, Cfg::SMEM_BYTES);
    }
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, tdbox, tdrem, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return DG_ERR_CUDA;
    }
    return DG_OK;
}

// Co-resident clusters of S CTAs of a split configuration (cached per
// device).  The split kernel keeps one tile per cluster, so a plan is only
// used when every cluster of the grid fits at once.
template <int BN, int STAGES, int KS, int NWG>
int query_max_clusters(int S)
{
    using Cfg = KernelConfig<BN, STAGES, KS, true, false, NWG>;
    auto kern = dg::fp8_gemm_kernel<BN, STAGES, KS, dg::kDense, true, false, false, NWG>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) !=
            cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(S * 16), 1, 1);
    cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(S);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    return n;
}

int max_active_clusters(const TileChoice &c, int S)
{
    static int cache[kMaxDevices][5] = {};  // S = 2, 4, 8, 16 (index log2(S))
    // The 128-column split tile of an N-major B uses a little less shared
    // memory than the 144-column one and runs one CTA per SM too: the same
    // clusters fit.
    if ((c.bn != 144 && c.bn != 128) || !c.split || S < 1)
        return 0;
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) {
        // no device (host-only planning, dg_describe_config): one CTA per SM
        const int cap = g_num_sms_cap.load();
        return (cap > 0 ? cap : 148) / S;
    }
    int idx = 0;
    while ((2 << idx) < S)
        ++idx;
    if (cache[dev][idx] == 0) {
        const int n = query_max_clusters<144, 3, 2, 3>(S);
        cache[dev][idx] = n > 0 ? n : -1;
    }
    // The SM cap (dg_set_num_sms) bounds the clusters too.
    const int cap = effective_sms(dev) / S;
    const int n = cache[dev][idx];
    return n < 0 ? 0 : (n < cap ? n : cap);
}

template <int LAYOUT, bool A_MN = false, bool B_MN = false>
dg_status_t dispatch(const Plan &plan, const void *A, uint64_t a_rows, const void *B,
                     uint64_t b_rows, GemmParams p, int sms, cudaStream_t stream)
{
    const TileChoice &c = plan.c;
    p.num_nb = (p.N + c.bn - 1) / c.bn;
    if ((A_MN || B_MN) && c.pair)
        return DG_ERR_UNSUPPORTED;  // the planner keeps MN-major operands on one-CTA tiles
    if (c.pair) {
        // the pair scheduler counts 256-row pair rows
        p.num_mb = (p.num_mb + 1) / 2;
        if (LAYOUT != dg::kMasked)
            p.raster = choose_raster(p.num_mb, 2 * dg::kBM, p.K);
        p.ksplit = 1;
        p.kb_per_split = p.num_kb;
        const int pairs = sms / 2;
        const int64_t ptiles = static_cast<int64_t>(p.num_mb) * p.num_nb;
        int grid_pairs = pairs;
        if (LAYOUT != dg::kMasked && ptiles < pairs)
            grid_pairs = static_cast<int>(ptiles);
        if (grid_pairs <= 0)
            return DG_OK;
        if (c.bn == 160 && c.stages == 3 && c.ks == 2 && c.wg == 2 && !c.rebal)
            return launch_pair<160, 3, 2, LAYOUT, 2>(A, a_rows, B, b_rows, p, 2 * grid_pairs, stream);
        if (c.bn == 160 && c.stages == 3 && c.ks == 2 && c.wg == 2 && c.rebal)
            return launch_pair<160, 3, 2, LAYOUT, 2, true>(A, a_rows, B, b_rows, p, 2 * grid_pairs, stream);
        if (c.bn == 160 && c.stages == 3 && c.ks == 2 && c.wg == 4)
            return launch_pair<160, 3, 2, LAYOUT, 4>(A, a_rows, B, b_rows, p, 2 * grid_pairs, stream);
        if (c.bn == 128 && c.stages == 4 && c.ks == 2 && c.wg == 2)
            return launch_pair<128, 4, 2, LAYOUT, 2>(A, a_rows, B, b_rows, p, 2 * grid_pairs, stream);
        if (c.bn == 192 && c.stages == 3 && c.ks == 2 && c.wg == 3)
            return launch_pair<192, 3, 2, LAYOUT, 3>(A, a_rows, B, b_rows, p, 2 * grid_pairs, stream);
        return DG_ERR_UNSUPPORTED;
    }
    p.ksplit = plan.ksplit;
    p.kb_per_split = (p.num_kb + plan.ksplit - 1) / plan.ksplit;
    const int64_t tiles = static_cast<int64_t>(LAYOUT == dg::kKGrouped ? p.G : 1) * p.num_mb * p.num_nb;
    if (plan.ksplit > 1) {
        const size_t bytes = static_cast<size_t>(tiles) * plan.ksplit * c.bn * dg::kBM * sizeof(float);
        void *ws = nullptr;
        const dg_status_t st = split_workspace(current_device(), bytes, &ws);
        if (st != DG_OK)
            return st;
        p.ws = static_cast<float *>(ws);
    }
    int grid = sms;
    if (plan.ksplit > 1)
        grid = static_cast<int>(tiles * plan.ksplit);
    else if (LAYOUT != dg::kMasked)
        grid = static_cast<int>(tiles < sms ? tiles : sms);
    if (grid <= 0)
        return DG_OK;
#define DG_TILE_CASE(BN_, ST_, KS_)                                                          \
    if constexpr (!B_MN || BN_ % 128 == 0) {                                                  \
        if (c.bn == BN_ && c.stages == ST_ && c.ks == KS_ && !c.split)                        \
            return launch_kernel<BN_, ST_, KS_, LAYOUT, false, A_MN, B_MN>(A, a_rows, B, b_rows, p, \
                                                                           grid, stream);     \
    }
    DG_TILE_CASE(112, 3, 2)
    DG_TILE_CASE(128, 5, 1)
    DG_TILE_CASE(224, 2, 2)
    DG_TILE_CASE(256, 3, 1)
    DG_TILE_CASE(256, 4, 1)
    if constexpr (LAYOUT == dg::kMasked && !A_MN && !B_MN) {
        // decode-sized groups; a second producer warp issues the B boxes
        if (c.bn == 128 && c.stages == 3 && c.ks == 2 && c.masked_only)
            return launch_kernel<128, 3, 2, LAYOUT, false, false, false, 2, true>(A, a_rows, B, b_rows, p,
                                                                                grid, stream);
    }
#undef DG_TILE_CASE
    if constexpr (LAYOUT == dg::kDense && !B_MN) {
        if (c.bn == 144 && c.stages == 3 && c.ks == 2 && c.split && c.wg == 3)
            return launch_kernel<144, 3, 2, LAYOUT, true, A_MN, false, 3>(A, a_rows, B, b_rows, p, grid,
                                                                          stream);
    }
    if constexpr (LAYOUT == dg::kDense && B_MN) {
        // an N-major B splits K on whole 128-column boxes
        if (c.bn == 128 && c.stages == 3 && c.ks == 2 && c.split && c.nmajor_split)
            return launch_kernel<128, 3, 2, LAYOUT, true, A_MN, true, 2>(A, a_rows, B, b_rows, p, grid,
                                                                         stream);
    }
    return DG_ERR_UNSUPPORTED;
}

dg_status_t check_common(const void *A, const float *sA, const void *B, const float *sB,
                         const void *D, int N, int K)
{
    if (!A || !sA || !B || !sB || !D)
        return DG_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0)
        return DG_ERR_INVALID_ARG;
    if (K % 128 != 0 || N % 16 != 0)
        return DG_ERR_UNSUPPORTED;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16) || !aligned(sA, 16) ||
        !aligned(sB, 4))
        return DG_ERR_ALIGNMENT;
    return DG_OK;
}

// The dense GEMM in any of the four operand layouts: A K-major ([M][K]) or
// M-major ([K][M], a_mn), B K-major ([N][K]) or N-major ([K][N], b_mn).
dg_status_t dense_gemm(const void *A, const float *sA, const void *B, const float *sB, void *D,
                       int M, int N, int K, bool a_mn, bool b_mn, cudaStream_t stream)
{
    if (M < 0)
        return DG_ERR_INVALID_ARG;
    dg_status_t st = check_common(A, sA, B, sB, D, N, K);
    if (st != DG_OK)
        return st;
    if (a_mn && M % 16 != 0)
        return DG_ERR_UNSUPPORTED;  // rows of an M-major A must be whole 16-byte units
    if (M == 0)
        return DG_OK;
    const int dev = current_device();
    const int sms = effective_sms(dev);
    if (sms <= 0)
        return DG_ERR_CUDA;
    GemmParams p{};
    p.sA = sA;
    p.sB = sB;
    p.D = static_cast<__nv_bfloat16 *>(D);
    p.M = M;
    p.N = N;
    p.K = K;
    p.G = 1;
    p.sa_ld = dg_get_tma_aligned_size(M, 4);
    p.num_kb = K / 128;
    p.nbn = (N + 127) / 128;
    p.num_mb = (M + 127) / 128;
    p.raster = choose_raster(p.num_mb, dg::kBM, K);
    p.timeout_ns = g_timeout_ns.load();
    p.stamps = g_stamps.load();
    p.stall_injection = g_stall_injection.load();
    const int limits = (a_mn || b_mn ? kNoPair : 0) | (b_mn ? kWholeBoxes : 0);
    const Plan plan = choose_plan(p.num_mb, (M + 255) / 256, N, p.num_kb, sms, true, limits);
    if (print_configs())
        std::fprintf(stderr, "[dg] dense %s%s M=%d N=%d K=%d -> BM=%d BN=%d stages=%d ks=%d ksplit=%d sms=%d\n",
                     a_mn ? "t" : "n", b_mn ? "n" : "t", M, N, K, plan.c.pair ? 256 : 128, plan.c.bn,
                     plan.c.stages, plan.c.ks, plan.ksplit, sms);
    const uint64_t am = static_cast<uint64_t>(M), bn = static_cast<uint64_t>(N);
    if (a_mn && b_mn)
        return dispatch<dg::kDense, true, true>(plan, A, am, B, bn, p, sms, stream);
    if (a_mn)
        return dispatch<dg::kDense, true, false>(plan, A, am, B, bn, p, sms, stream);
    if (b_mn)
        return dispatch<dg::kDense, false, true>(plan, A, am, B, bn, p, sms, stream);
    return dispatch<dg::kDense>(plan, A, am, B, bn, p, sms, stream);
}

// ------------------------------------------------ UE8M0 block-scaled mode

// Tile shapes of the block-scaled kernels.  The tensor core applies the
// scales, so a tile's time is its MMA time (proportional to BN) plus a fixed
// fill/epilogue part: cost = waves x (BN + 48) x feed, where feed > 1 for
// one-CTA tiles, whose operand bytes per SM and K block ((128 + BN) x 128)
// approach the L2 -> SM limit at full MMA rate; pair tiles (256 x BN on two
// SMs, (128 + BN/2) x 128 bytes per SM) are taken when they fill every SM
// pair.  dg_set_tile_family restricts the family as for the fp32-scale mode.
struct BsChoice {
    int bn, stages, ks, pair;
    double feed;
    int ksplit = 1;  // > 1: the dense K-split kernel, a cluster of ksplit CTAs per tile
};

// The dense decode plan of the UE8M0 mode: problems with too few tiles to
// fill the GPU and a long K range (at least 16 K blocks: below that the
// cluster barrier and the reduction cost more than the split saves, e.g.
// 16.4 vs 11.1 us on 128 x 256 x 512) split each 128 x 144 tile's K range
// over a cluster of S CTAs (S = 8, 4 or 2: the largest that leaves every
// split two K blocks and keeps all of the grid's clusters co-resident).
constexpr int kBsSplitMinKb = 16;
constexpr int kBsSplitBN = 144;
int bs_split_max_clusters(int S);
constexpr BsChoice kBsChoices[] = {
    {128, 3, 2, 0, 1.25}, {160, 2, 2, 0, 1.25}, {192, 2, 2, 0, 1.25}, {224, 2, 2, 0, 1.25},
    {128, 4, 2, 1, 1.0},  {160, 3, 2, 1, 1.0},  {192, 3, 2, 1, 1.0},  {224, 3, 2, 1, 1.0},
};

BsChoice choose_bs(int64_t m_blocks, int64_t pair_rows, int N, int sms)
{
    BsChoice best = kBsChoices[0];
    double best_cost = 1e300;
    for (const BsChoice &c : kBsChoices) {
        if (forced_block_n() > 0 && c.bn != forced_block_n())
            continue;
        if (forced_pair() >= 0 && c.pair != forced_pair())
            continue;
        const int units = c.pair ? sms / 2 : sms;
        if (units <= 0)
            continue;
        const int64_t tiles = (c.pair ? pair_rows : m_blocks) * ((N + c.bn - 1) / c.bn);
        if (c.pair && tiles < units && forced_pair() != 1)
            continue;
        const int64_t waves = (tiles + units - 1) / units;
        const double cost = static_cast<double>(waves) * (c.bn + 48) * c.feed;
        if (cost < best_cost) {
            best_cost = cost;
            best = c;
        }
    }
    return best;
}

BsChoice choose_bs_dense(int64_t m_blocks, int64_t pair_rows, int N, int num_kb, int sms)
{
    BsChoice c = choose_bs(m_blocks, pair_rows, N, sms);
    if (forced_block_n() > 0 || forced_pair() == 1)
        return c;
    const int64_t tiles = m_blocks * ((N + c.bn - 1) / c.bn);
    if (c.pair || tiles * 2 > sms || num_kb < kBsSplitMinKb)
        return c;
    const int64_t split_tiles = m_blocks * ((N + kBsSplitBN - 1) / kBsSplitBN);
    for (int S = 8; S >= 2; S /= 2) {
        const int kbps = (num_kb + S - 1) / S;
        if (kbps < 2 || (num_kb + kbps - 1) / kbps != S)
            continue;
        if (split_tiles > bs_split_max_clusters(S))
            continue;
        BsChoice sc{kBsSplitBN, 3, 2, 0, 1.0, S};
        return sc;
    }
    return c;
}

// Masked (decode) problems are HBM-bound: the one-CTA 128-column tile, whose
// three-stage ring keeps the most bytes in flight, measured best (129 us on
// 16 x 256 x 4096 x 7168 against 140-162 us for the other shapes); an
// explicit tile-family or width restriction still goes through choose_bs.
BsChoice choose_bs_masked(int64_t m_blocks, int64_t pair_rows, int N, int sms)
{
    if (forced_block_n() <= 0 && forced_pair() < 0)
        return kBsChoices[0];
    return choose_bs(m_blocks, pair_rows, N, sms);
}

template <int BN, int STAGES, int KS, int LAYOUT, bool PAIR, bool SPLIT = false>
dg_status_t launch_bs(const void *A, uint64_t a_rows, const void *B, uint64_t b_rows, const GemmParams &p,
                      int grid, cudaStream_t stream)
{
    using Cfg = dg::BsConfig<BN, STAGES, KS, PAIR, SPLIT>;
    CUtensorMap ta, tb, td64, tdrem;
    if (!make_tmap_operand(&ta, A, static_cast<uint64_t>(p.K), a_rows, dg::kBM, KS) ||
        !make_tmap_operand(&tb, B, static_cast<uint64_t>(p.K), b_rows, Cfg::B_ROWS, KS))
        return DG_ERR_CUDA;
    if (!make_tmap_bf16(&td64, p.D, static_cast<uint64_t>(p.N), a_rows, 64, dg::kBM,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return DG_ERR_CUDA;
    if (Cfg::EPI_REM > 0) {
        if (!make_tmap_bf16(&tdrem, p.D, static_cast<uint64_t>(p.N), a_rows, Cfg::EPI_REM, dg::kBM,
                            CU_TENSOR_MAP_SWIZZLE_NONE))
            return DG_ERR_CUDA;
    } else {
        tdrem = td64;
    }
    if (SPLIT && p.ksplit >= 2 && dg::kBM % p.ksplit == 0) {
        // the K-split reduction's maps: the partials and one CTA's output rows
        const int rows_per = dg::kBM / p.ksplit;
        const uint64_t tiles = static_cast<uint64_t>(p.num_mb) * static_cast<uint64_t>(p.num_nb);
        if (!make_tmap_split_ws(&td64, p.ws, BN, p.ksplit, tiles, rows_per) ||
            !make_tmap_bf16(&tdrem, p.D, static_cast<uint64_t>(p.N), a_rows, BN, rows_per,
                            CU_TENSOR_MAP_SWIZZLE_NONE))
            return DG_ERR_CUDA;
    }
    auto kern = dg::fp8_gemm_bs_kernel<BN, STAGES, KS, LAYOUT, PAIR, SPLIT>;
    static std::atomic<bool> attr_set[kMaxDevices];
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices)
        return DG_ERR_CUDA;
    if (!attr_set[dev].load()) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) !=
            cudaSuccess)
            return DG_ERR_CUDA;
        attr_set[dev].store(true);
    }
    cudaLaunchConfig_t cfg = {};
    // the K split runs a 3-D grid (split, column tile, 128-row block)
    cfg.gridDim = SPLIT ? dim3(static_cast<unsigned>(p.ksplit), static_cast<unsigned>(p.num_nb),
                               static_cast<unsigned>(p.num_mb))
                        : dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = PAIR ? 2u : (SPLIT ? static_cast<unsigned>(p.ksplit) : 1u);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (PAIR || SPLIT) ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, td64, tdrem, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return DG_ERR_CUDA;
    }
    return DG_OK;
}

// Co-resident clusters of S CTAs of the UE8M0 split kernel (cached per
// device, bounded by the SM cap).
int bs_split_max_clusters(int S)
{
    static int cache[kMaxDevices][4] = {};  // S = 2, 4, 8 (index log2(S) - 1)
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices || S < 2 || S > 8)
        return 0;
    const int idx = S == 2 ? 0 : (S == 4 ? 1 : 2);
    if (cache[dev][idx] == 0) {
        using Cfg = dg::BsConfig<kBsSplitBN, 3, 2, false, true>;
        auto kern = dg::fp8_gemm_bs_kernel<kBsSplitBN, 3, 2, dg::kDense, false, true>;
        int n = 0;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) ==
            cudaSuccess) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(static_cast<unsigned>(S * 16), 1, 1);
            cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
            cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = static_cast<unsigned>(S);
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess)
                n = 0;
        }
        (void)cudaGetLastError();
        cache[dev][idx] = n > 0 ? n : -1;
    }
    const int cap = effective_sms(dev) / S;
    const int n = cache[dev][idx];
    return n < 0 ? 0 : (n < cap ? n : cap);
}

template <int LAYOUT>
dg_status_t dispatch_bs(const BsChoice &c, const void *A, uint64_t a_rows, const void *B, uint64_t b_rows,
                        GemmParams p, int sms, cudaStream_t stream)
{
    p.num_nb = (p.N + c.bn - 1) / c.bn;
    p.ksplit = 1;
    p.kb_per_split = p.num_kb;
    if constexpr (LAYOUT == dg::kDense) {
        if (c.ksplit > 1) {
            // one tile per cluster of ksplit CTAs; fp32 partials in the workspace
            p.ksplit = c.ksplit;
            p.kb_per_split = (p.num_kb + c.ksplit - 1) / c.ksplit;
            const int64_t tiles = static_cast<int64_t>(p.num_mb) * p.num_nb;
            const size_t bytes = static_cast<size_t>(tiles) * c.ksplit * c.bn * dg::kBM * sizeof(float);
            void *ws = nullptr;
            const dg_status_t st = split_workspace(current_device(), bytes, &ws);
            if (st != DG_OK)
                return st;
            p.ws = static_cast<float *>(ws);
            if (c.bn == kBsSplitBN && c.stages == 3 && c.ks == 2)
                return launch_bs<kBsSplitBN, 3, 2, LAYOUT, false, true>(A, a_rows, B, b_rows, p,
                                                                       static_cast<int>(tiles * c.ksplit), stream);
            return DG_ERR_UNSUPPORTED;
        }
    }
    if (c.pair) {
        // the pair scheduler counts 256-row pair rows
        p.num_mb = (p.num_mb + 1) / 2;
        if (LAYOUT != dg::kMasked)
            p.raster = choose_raster(p.num_mb, 2 * dg::kBM, p.K);
        const int pairs = sms / 2;
        const int64_t ptiles = static_cast<int64_t>(p.num_mb) * p.num_nb;
        int grid_pairs = pairs;
        if (LAYOUT != dg::kMasked && ptiles < pairs)
            grid_pairs = static_cast<int>(ptiles);
        if (grid_pairs <= 0)
            return DG_OK;
#define DG_BS_PAIR_CASE(BN_, ST_, KS_)                                                              \
        if (c.bn == BN_ && c.stages == ST_ && c.ks == KS_)                                           \
            return launch_bs<BN_, ST_, KS_, LAYOUT, true>(A, a_rows, B, b_rows, p, 2 * grid_pairs, stream);
        DG_BS_PAIR_CASE(128, 4, 2)
        DG_BS_PAIR_CASE(160, 3, 2)
        DG_BS_PAIR_CASE(192, 3, 2)
        DG_BS_PAIR_CASE(224, 3, 2)
#undef DG_BS_PAIR_CASE
        return DG_ERR_UNSUPPORTED;
    }
    const int64_t tiles = static_cast<int64_t>(p.num_mb) * p.num_nb;
    int grid = sms;
    if (LAYOUT != dg::kMasked)
        grid = static_cast<int>(tiles < sms ? tiles : sms);
    if (grid <= 0)
        return DG_OK;
#define DG_BS_CASE(BN_, ST_, KS_)                                                                   \
    if (c.bn == BN_ && c.stages == ST_ && c.ks == KS_)                                               \
        return launch_bs<BN_, ST_, KS_, LAYOUT, false>(A, a_rows, B, b_rows, p, grid, stream);
    DG_BS_CASE(128, 3, 2)
    DG_BS_CASE(160, 2, 2)
    DG_BS_CASE(192, 2, 2)
    DG_BS_CASE(224, 2, 2)
#undef DG_BS_CASE
    return DG_ERR_UNSUPPORTED;
}

dg_status_t check_bs(const void *A, const int32_t *sfa, const void *B, const int32_t *sfb, const void *D,
                     int N, int K)
{
    if (!A || !sfa || !B || !sfb || !D)
        return DG_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0)
        return DG_ERR_INVALID_ARG;
    if (K % 128 != 0 || N % 16 != 0)
        return DG_ERR_UNSUPPORTED;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16) || !aligned(sfa, 16) || !aligned(sfb, 4))
        return DG_ERR_ALIGNMENT;
    return DG_OK;
}

// Parameters shared by the three layouts of the block-scaled mode.
GemmParams bs_params(const int32_t *sfa, const int32_t *sfb, void *D, int M, int N, int K, int G)
{
    GemmParams p{};
    p.sfa = sfa;
    p.sfb = sfb;
    p.D = static_cast<__nv_bfloat16 *>(D);
    p.M = M;
    p.N = N;
    p.K = K;
    p.G = G;
    p.sfa_ld = dg_get_tma_aligned_size(M, 4);
    p.num_kb = K / 128;
    p.num_kg = (p.num_kb + 3) / 4;
    p.nbn = (N + 127) / 128;
    p.num_mb = (M + 127) / 128;
    p.raster = choose_raster(p.num_mb, dg::kBM, K);
    p.timeout_ns = g_timeout_ns.load();
    p.stamps = g_stamps.load();
    p.stall_injection = g_stall_injection.load();
    return p;
}

// Fixed scratch of dg_fp8_gemm_nt_noalloc and the tile width of the K-split
// kernel it runs.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr int kNoAllocBN = 144;
int noalloc_split(int M, int N, int K, int sms);

}  // namespace

// =================================================================== C ABI

extern "C" {

dg_status_t dg_fp8_gemm_nt(const void *A, const float *sA, const void *B, const float *sB,
                           void *D, int M, int N, int K, cudaStream_t stream)
{
    return dense_gemm(A, sA, B, sB, D, M, N, K, false, false, stream);
}

dg_status_t dg_fp8_gemm_nn(const void *A, const float *sA, const void *B, const float *sB,
                           void *D, int M, int N, int K, cudaStream_t stream)
{
    return dense_gemm(A, sA, B, sB, D, M, N, K, false, true, stream);
}

dg_status_t dg_fp8_gemm_tn(const void *A, const float *sA, const void *B, const float *sB,
                           void *D, int M, int N, int K, cudaStream_t stream)
{
    return dense_gemm(A, sA, B, sB, D, M, N, K, true, true, stream);
}

dg_status_t dg_fp8_gemm_tt(const void *A, const float *sA, const void *B, const float *sB,
                           void *D, int M, int N, int K, cudaStream_t stream)
{
    return dense_gemm(A, sA, B, sB, D, M, N, K, true, false, stream);
}

dg_status_t dg_fp8_k_grouped_gemm_tn_contiguous(const void *A, const float *sA, const void *B,
                                                const float *sB, float *D, const int32_t *k_offsets,
                                                int M, int N, int K, int num_groups, cudaStream_t stream)
{
    if (!A || !sA || !B || !sB || !D || !k_offsets || M < 0 || N <= 0 || K < 0 || num_groups <= 0)
        return DG_ERR_INVALID_ARG;
    if (K % 128 != 0 || N % 16 != 0 || M % 16 != 0)
        return DG_ERR_UNSUPPORTED;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16) || !aligned(sA, 16) ||
        !aligned(sB, 16) || !aligned(k_offsets, 4))
        return DG_ERR_ALIGNMENT;
    if (static_cast<int64_t>(num_groups) * M * N > 0x7FFFFFFFll * 4)
        return DG_ERR_UNSUPPORTED;
    if (M == 0)
        return DG_OK;
    if (K == 0) {
        // every group is empty: each D_g is zero
        if (cudaMemsetAsync(D, 0, static_cast<size_t>(num_groups) * M * N * sizeof(float), stream) !=
            cudaSuccess) {
            (void)cudaGetLastError();
            return DG_ERR_CUDA;
        }
        return DG_OK;
    }
    const int dev = current_device();
    const int sms = effective_sms(dev);
    if (sms <= 0)
        return DG_ERR_CUDA;
    GemmParams p{};
    p.sA = sA;
    p.sB = sB;
    p.D = reinterpret_cast<__nv_bfloat16 *>(D);  // shapes the unused store tensor maps only
    p.D32 = D;
    p.k_offsets = k_offsets;
    p.M = M;
    p.N = N;
    p.K = K;
    p.G = num_groups;
    p.sa_ld = dg_get_tma_aligned_size(M, 4);
    p.num_kb = K / 128;
    p.nbn = (N + 127) / 128;
    p.num_mb = (M + 127) / 128;
    p.raster = 1;
    p.timeout_ns = g_timeout_ns.load();
    p.stamps = g_stamps.load();
    p.stall_injection = g_stall_injection.load();
    const int avg_kb = p.num_kb / num_groups > 0 ? p.num_kb / num_groups : 1;
    const Plan plan = choose_plan(static_cast<int64_t>(num_groups) * p.num_mb, 0, N, avg_kb, sms, false,
                                  kNoPair | kWholeBoxes);
    if (print_configs())
        std::fprintf(stderr, "[dg] k-grouped tn G=%d M=%d N=%d K=%d -> BM=128 BN=%d stages=%d ks=%d sms=%d\n",
                     num_groups, M, N, K, plan.c.bn, plan.c.stages, plan.c.ks, sms);
    return dispatch<dg::kKGrouped, true, true>(plan, A, static_cast<uint64_t>(M), B,
                                                static_cast<uint64_t>(N), p, sms, stream);
}

dg_status_t dg_fp8_gemm_nt_acc(const void *A, const float *sA, const void *B, const float *sB,
                               const float *C, float *D, int M, int N, int K, cudaStream_t stream)
{
    if (M < 0 || !C)
        return DG_ERR_INVALID_ARG;
    dg_status_t st = check_common(A, sA, B, sB, D, N, K);
    if (st != DG_OK)
        return st;
    if (!aligned(C, 16))
        return DG_ERR_ALIGNMENT;
    if (M == 0)
        return DG_OK;
    const int dev = current_device();
    const int sms = effective_sms(dev);
    if (sms <= 0)
        return DG_ERR_CUDA;
    GemmParams p{};
    p.sA = sA;
    p.sB = sB;
    // The bf16 output pointer only shapes the (unused) store tensor maps;
    // the kernels write D through D32.
    p.D = reinterpret_cast<__nv_bfloat16 *>(D);
    p.C = C;
    p.D32 = D;
    p.M = M;
    p.N = N;
    p.K = K;
    p.G = 1;
    p.sa_ld = dg_get_tma_aligned_size(M, 4);
    p.num_kb = K / 128;
    p.nbn = (N + 127) / 128;
    p.num_mb = (M + 127) / 128;
    p.raster = choose_raster(p.num_mb, dg::kBM, K);
    p.timeout_ns = g_timeout_ns.load();
    p.stamps = g_stamps.load();
    p.stall_injection = g_stall_injection.load();
    const Plan plan = choose_plan(p.num_mb, (M + 255) / 256, N, p.num_kb, sms, true);
    if (print_configs())
        std::fprintf(stderr, "[dg] dense accumulate M=%d N=%d K=%d -> BM=%d BN=%d stages=%d ks=%d ksplit=%d sms=%d\n",
                     M, N, K, plan.c.pair ? 256 : 128, plan.c.bn, plan.c.stages, plan.c.ks, plan.ksplit, sms);
    return dispatch<dg::kDense>(plan, A, static_cast<uint64_t>(M), B, static_cast<uint64_t>(N), p,
                                sms, stream);
}

dg_status_t dg_fp8_grouped_gemm_contiguous(const void *A, const float *sA, const void *B,
                                           const float *sB, void *D, const int32_t *m_indices,
                                           int M_total, int N, int K, int num_groups,
                                           cudaStream_t stream)
{
    if (M_total < 0 || num_groups <= 0 || !m_indices)
        return DG_ERR_INVALID_ARG;
    dg_status_t st = check_common(A, sA, B, sB, D, N, K);
    if (st != DG_OK)
        return st;
    if (M_total % 128 != 0)
        return DG_ERR_UNSUPPORTED;
    if (!aligned(m_indices, 4))
        return DG_ERR_ALIGNMENT;
    if (M_total == 0)
        return DG_OK;
    if (static_cast<int64_t>(num_groups) * N > 0x7FFFFFFF)
        return DG_ERR_UNSUPPORTED;
    const int dev = current_device();
    const int sms = effective_sms(dev);
    if (sms <= 0)
        return DG_ERR_CUDA;
    GemmParams p{};
    p.sA = sA;
    p.sB = sB;
    p.D = static_cast<__nv_bfloat16 *>(D);
    p.m_indices = m_indices;
    p.M = M_total;
    p.N = N;
    p.K = K;
    p.G = num_groups;
    p.sa_ld = dg_get_tma_aligned_size(M_total, 4);
    p.num_kb = K / 128;
    p.nbn = (N + 127) / 128;
    p.num_mb = M_total / 128;
    p.raster = choose_raster(p.num_mb, dg::kBM, K);
    p.timeout_ns = g_timeout_ns.load();
    p.stamps = g_stamps.load();
    p.stall_injection = g_stall_injection.load();
    const Plan plan = choose_plan(p.num_mb, (M_total + 255) / 256, N, p.num_kb, sms, false);
    if (print_configs())
        std::fprintf(stderr, "[dg] contiguous M=%d N=%d K=%d G=%d -> BM=%d BN=%d stages=%d ks=%d sms=%d\n",
                     M_total, N, K, num_groups, plan.c.pair ? 256 : 128, plan.c.bn, plan.c.stages,
                     plan.c.ks, sms);
    return dispatch<dg::kContiguous>(plan, A, static_cast<uint64_t>(M_total), B,
                                     static_cast<uint64_t>(num_groups) * N, p, sms, stream);
}

dg_status_t dg_fp8_grouped_gemm_masked(const void *A, const float *sA, const void *B,
                                       const float *sB, void *D, const int32_t *masked_m,
                                       int num_groups, int max_m, int N, int K, int expected_m,
                                       cudaStream_t stream)
{
    if (num_groups <= 0 || max_m < 0 || expected_m < 0 || !masked_m)
        return DG_ERR_INVALID_ARG;
    dg_status_t st = check_common(A, sA, B, sB, D, N, K);
    if (st != DG_OK)
        return st;
    if (!aligned(masked_m, 4))
        return DG_ERR_ALIGNMENT;
    if (max_m == 0)
        return DG_OK;
    if (static_cast<int64_t>(num_groups) * max_m > 0x7FFFFFFF ||
        static_cast<int64_t>(num_groups) * N > 0x7FFFFFFF)
        return DG_ERR_UNSUPPORTED;
    const int dev = current_device();
    const int sms = effective_sms(dev);
    if (sms <= 0)
        return DG_ERR_CUDA;
    GemmParams p{};
    p.sA = sA;
    p.sB = sB;
    p.D = static_cast<__nv_bfloat16 *>(D);
    p.masked_m = masked_m;
    p.M = max_m;
    p.N = N;
    p.K = K;
    p.G = num_groups;
    p.sa_ld = dg_get_tma_aligned_size(max_m, 4);
    p.num_kb = K / 128;
    p.nbn = (N + 127) / 128;
    p.num_mb = (max_m + 127) / 128;
    p.raster = 1;
    p.timeout_ns = g_timeout_ns.load();
    p.stamps = g_stamps.load();
    p.stall_injection = g_stall_injection.load();
    const int em = (expected_m > 0 && expected_m < max_m) ? expected_m : max_m;
    Plan plan = choose_plan(static_cast<int64_t>(num_groups) * ((em + 127) / 128),
                            static_cast<int64_t>(num_groups) * ((em + 255) / 256), N, p.num_kb, sms, false);
    // Decode-sized groups (at most two 128-row blocks each) make the problem
    // HBM-bound on the weights: the 128-column one-CTA tile with three
    // stages of two K blocks keeps six K blocks in flight per SM with half
    // the TMA instructions of one-K-block stages, its A and B boxes issued by
    // two producer warps, and measured best (16 x 256 x 4096 x 7168: 144 us,
    // against 156 us with one producer warp, 172 us for five one-K-block
    // stages and 171-176 us for 112, 224 and 256 columns), unless a tile
    // width or family is pinned.
    if (em <= 2 * dg::kBM && forced_block_n() <= 0 && forced_pair() < 0)
        plan = Plan{kTileChoices[kMaskedDecodeTile], 1};
    if (print_configs())
        std::fprintf(stderr,
                     "[dg] masked G=%d max_m=%d expected_m=%d N=%d K=%d -> BM=%d BN=%d stages=%d ks=%d sms=%d\n",
                     num_groups, max_m, em, N, K, plan.c.pair ? 256 : 128, plan.c.bn, plan.c.stages,
                     plan.c.ks, sms);
    return dispatch<dg::kMasked>(plan, A, static_cast<uint64_t>(num_groups) * max_m, B,
                                 static_cast<uint64_t>(num_groups) * N, p, sms, stream);
}

dg_status_t dg_fp8_gemm_nt_ue8m0(const void *A, const int32_t *sfa, const void *B, const int32_t *sfb,
                                 void *D, int M, int N, int K, cudaStream_t stream)
{
    if (M < 0)
        return DG_ERR_INVALID_ARG;
    dg_status_t st = check_bs(A, sfa, B, sfb, D, N, K);
    if (st != DG_OK)
        return st;
    if (M == 0)
        return DG_OK;
    const int sms = effective_sms(current_device());
    if (sms <= 0)
        return DG_ERR_CUDA;
    GemmParams p = bs_params(sfa, sfb, D, M, N, K, 1);
    const BsChoice c = choose_bs_dense(p.num_mb, (M + 255) / 256, N, p.num_kb, sms);
    if (print_configs())
        std::fprintf(stderr, "[dg] dense ue8m0 M=%d N=%d K=%d -> BM=%d BN=%d stages=%d ks=%d ksplit=%d sms=%d\n",
                     M, N, K, c.pair ? 256 : 128, c.bn, c.stages, c.ks, c.ksplit, sms);
    return dispatch_bs<dg::kDense>(c, A, static_cast<uint64_t>(M), B, static_cast<uint64_t>(N), p, sms,
                                   stream);
}

dg_status_t dg_fp8_grouped_gemm_contiguous_ue8m0(const void *A, const int32_t *sfa, const void *B,
                                                 const int32_t *sfb, void *D, const int32_t *m_indices,
                                                 int M_total, int N, int K, int num_groups,
                                                 cudaStream_t stream)
{
    if (M_total < 0 || num_groups <= 0 || !m_indices)
        return DG_ERR_INVALID_ARG;
    dg_status_t st = check_bs(A, sfa, B, sfb, D, N, K);
    if (st != DG_OK)
        return st;
    if (M_total % 128 != 0)
        return DG_ERR_UNSUPPORTED;
    if (!aligned(m_indices, 4))
        return DG_ERR_ALIGNMENT;
    if (M_total == 0)
        return DG_OK;
    if (static_cast<int64_t>(num_groups) * N > 0x7FFFFFFF)
        return DG_ERR_UNSUPPORTED;
    const int sms = effective_sms(current_device());
    if (sms <= 0)
        return DG_ERR_CUDA;
    GemmParams p = bs_params(sfa, sfb, D, M_total, N, K, num_groups);
    p.m_indices = m_indices;
    const BsChoice c = choose_bs(p.num_mb, (M_total + 255) / 256, N, sms);
    if (print_configs())
        std::fprintf(stderr, "[dg] contiguous ue8m0 M=%d N=%d K=%d G=%d -> BM=%d BN=%d stages=%d ks=%d sms=%d\n",
                     M_total, N, K, num_groups, c.pair ? 256 : 128, c.bn, c.stages, c.ks, sms);
    return dispatch_bs<dg::kContiguous>(c, A, static_cast<uint64_t>(M_total), B,
                                        static_cast<uint64_t>(num_groups) * N, p, sms, stream);
}

dg_status_t dg_fp8_grouped_gemm_masked_ue8m0(const void *A, const int32_t *sfa, const void *B,
                                             const int32_t *sfb, void *D, const int32_t *masked_m,
                                             int num_groups, int max_m, int N, int K, int expected_m,
                                             cudaStream_t stream)
{
    if (num_groups <= 0 || max_m < 0 || expected_m < 0 || !masked_m)
        return DG_ERR_INVALID_ARG;
    dg_status_t st = check_bs(A, sfa, B, sfb, D, N, K);
    if (st != DG_OK)
        return st;
    if (!aligned(masked_m, 4))
        return DG_ERR_ALIGNMENT;
    if (max_m == 0)
        return DG_OK;
    if (static_cast<int64_t>(num_groups) * max_m > 0x7FFFFFFF ||
        static_cast<int64_t>(num_groups) * N > 0x7FFFFFFF)
        return DG_ERR_UNSUPPORTED;
    const int sms = effective_sms(current_device());
    if (sms <= 0)
        return DG_ERR_CUDA;
    GemmParams p = bs_params(sfa, sfb, D, max_m, N, K, num_groups);
    p.masked_m = masked_m;
    p.raster = 1;
    const int em = (expected_m > 0 && expected_m < max_m) ? expected_m : max_m;
    const BsChoice c = choose_bs_masked(static_cast<int64_t>(num_groups) * ((em + 127) / 128),
                                        static_cast<int64_t>(num_groups) * ((em + 255) / 256), N, sms);
    if (print_configs())
        std::fprintf(stderr,
                     "[dg] masked ue8m0 G=%d max_m=%d expected_m=%d N=%d K=%d -> BM=%d BN=%d stages=%d ks=%d sms=%d\n",
                     num_groups, max_m, em, N, K, c.pair ? 256 : 128, c.bn, c.stages, c.ks, sms);
    return dispatch_bs<dg::kMasked>(c, A, static_cast<uint64_t>(num_groups) * max_m, B,
                                    static_cast<uint64_t>(num_groups) * N, p, sms, stream);
}

dg_status_t dg_transform_sf_ue8m0(const float *sf, int32_t *out, int rows, int K, int batch, int mn_major,
                                  cudaStream_t stream)
{
    if (!sf || !out || rows < 0 || K <= 0 || batch <= 0 || (mn_major != 0 && mn_major != 1))
        return DG_ERR_INVALID_ARG;
    if (K % 128 != 0)
        return DG_ERR_UNSUPPORTED;
    if (!aligned(sf, 4) || !aligned(out, 4))
        return DG_ERR_ALIGNMENT;
    if (rows == 0)
        return DG_OK;
    const int out_ld = mn_major ? dg_get_tma_aligned_size(rows, 4) : rows;
    const int nkb = K / 128;
    const int64_t total = static_cast<int64_t>(batch) * ((nkb + 3) / 4) * out_ld;
    const int threads = 256;
    const int64_t want = (total + threads - 1) / threads;
    const int blocks = static_cast<int>(want < 4096 ? want : 4096);
    dg::transform_sf_ue8m0_kernel<<<blocks, threads, 0, stream>>>(sf, out, rows, out_ld, nkb, batch, mn_major);
    if (cudaPeekAtLastError() != cudaSuccess) {
        (void)cudaGetLastError();
        return DG_ERR_CUDA;
    }
    return DG_OK;
}

int dg_get_mk_alignment_for_contiguous_layout(void) { return 128; }

int dg_get_tma_aligned_size(int x, int elem_bytes)
{
    if (x < 0 || !(elem_bytes == 1 || elem_bytes == 2 || elem_bytes == 4 || elem_bytes == 8 ||
                   elem_bytes == 16))
        return -1;
    const int per = 16 / elem_bytes;
    return (x + per - 1) / per * per;
}

dg_status_t dg_set_num_sms(int n)
{
    if (n < 0)
        return DG_ERR_INVALID_ARG;
    g_num_sms_cap.store(n);
    return DG_OK;
}

int dg_get_num_sms(void) { return effective_sms(current_device()); }

dg_status_t dg_set_tile_family(int family)
{
    if (family < DG_TILES_AUTO || family > DG_TILES_PAIR)
        return DG_ERR_INVALID_ARG;
    g_forced_pair.store(family == DG_TILES_AUTO ? -1 : (family == DG_TILES_PAIR ? 1 : 0));
    return DG_OK;
}

dg_status_t dg_set_block_n(int n)
{
    bool known = n == 0;
    for (const TileChoice &c : kTileChoices)
        known = known || c.bn == n;
    for (const BsChoice &c : kBsChoices)
        known = known || c.bn == n;
    if (!known)
        return DG_ERR_INVALID_ARG;
    g_forced_bn.store(n);
    return DG_OK;
}

unsigned long long dg_get_tensor_map_encodes(void) { return g_tmap_encodes.load(); }

unsigned long long dg_get_device_allocations(void) { return g_device_allocs.load(); }

dg_status_t dg_set_timing_stamps(unsigned long long *stamps)
{
    if (stamps != nullptr && !aligned(stamps, 8))
        return DG_ERR_ALIGNMENT;
    g_stamps.store(stamps);
    return DG_OK;
}

dg_status_t dg_set_wait_timeout_ns(uint64_t ns)
{
    g_timeout_ns.store(ns == 0 ? kDefaultTimeoutNs : ns);
    return DG_OK;
}

dg_status_t dg_set_stall_injection(int enable)
{
    g_stall_injection.store(enable ? 1 : 0);
    return DG_OK;
}

dg_status_t dg_get_device_status_detail(cudaStream_t stream, uint32_t *word)
{
    if (!word)
        return DG_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(stream) != cudaSuccess)
        return DG_ERR_CUDA;
    unsigned int w = 0;
    if (cudaMemcpyFromSymbol(&w, dg::g_status_word, sizeof(w)) != cudaSuccess)
        return DG_ERR_CUDA;
    *word = w;
    return static_cast<dg_status_t>(w & 0xFF);
}

dg_status_t dg_get_device_status(cudaStream_t stream)
{
    uint32_t w = 0;
    dg_status_t st = dg_get_device_status_detail(stream, &w);
    if (st == DG_ERR_CUDA || st == DG_ERR_INVALID_ARG)
        return st;
    if (w != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(dg::g_status_word, &zero, sizeof(zero)) != cudaSuccess)
            return DG_ERR_CUDA;
    }
    return static_cast<dg_status_t>(w & 0xFF);
}

int dg_describe_config(int layout, int M, int N, int K, int groups, char *buf, int len)
{
    if (layout < 0 || layout > 6 || M < 0 || N <= 0 || K <= 0 || groups <= 0 || (len > 0 && !buf))
        return -1;
    // Without a device (host-only use) the SM cap alone decides, else 148.
    const int dev = current_device();
    int sms = effective_sms(dev);
    if (sms <= 0)
        sms = g_num_sms_cap.load() > 0 ? g_num_sms_cap.load() : 148;
    if (layout == 6) {
        // the dense GEMM through dg_fp8_gemm_nt_noalloc (ksplit=0: too large
        // for its fixed scratch)
        return std::snprintf(buf, len > 0 ? static_cast<size_t>(len) : 0,
                             "layout=6 BM=128 BN=%d BK=128 stages=3 ks=2 ksplit=%d pair=0 wg=2 sms=%d m_blocks=%d n_blocks=%d noalloc=1",
                             kNoAllocBN, noalloc_split(M, N, K - K % 128, sms), sms, (M + 127) / 128,
                             (N + kNoAllocBN - 1) / kNoAllocBN);
    }
    if (layout >= 3) {
        // the UE8M0 block-scaled mode (one-CTA or pair tiles, no K split)
        const int64_t mb = static_cast<int64_t>((M + 127) / 128) * (layout == 5 ? groups : 1);
        const int64_t pr = static_cast<int64_t>((M + 255) / 256) * (layout == 5 ? groups : 1);
        const BsChoice c = layout == 5   ? choose_bs_masked(mb, pr, N, sms)
                           : layout == 3 ? choose_bs_dense(mb, pr, N, K / 128 > 0 ? K / 128 : 1, sms)
                                         : choose_bs(mb, pr, N, sms);
        return std::snprintf(buf, len > 0 ? static_cast<size_t>(len) : 0,
                             "layout=%d BM=%d BN=%d BK=128 stages=%d ks=%d ksplit=%d pair=%d wg=1 sms=%d m_blocks=%lld n_blocks=%d ue8m0=1",
                             layout, c.pair ? 256 : 128, c.bn, c.stages, c.ks, c.ksplit, c.pair, sms,
                             static_cast<long long>(c.pair ? pr : mb), (N + c.bn - 1) / c.bn);
    }
    int64_t m_blocks = (M + 127) / 128;
    int64_t pair_rows = (M + 255) / 256;
    if (layout == 2) {
        m_blocks *= groups;
        pair_rows *= groups;
    }
    Plan plan = choose_plan(m_blocks, pair_rows, N, K / 128 > 0 ? K / 128 : 1, sms, layout == 0);
    if (layout == 2 && M <= 2 * dg::kBM && forced_block_n() <= 0 && forced_pair() < 0)
        plan = Plan{kTileChoices[kMaskedDecodeTile], 1};  // as dg_fp8_grouped_gemm_masked: decode-sized groups
    const TileChoice &c = plan.c;
    return std::snprintf(buf, len > 0 ? static_cast<size_t>(len) : 0,
                         "layout=%d BM=%d BN=%d BK=128 stages=%d ks=%d ksplit=%d pair=%d wg=%d sms=%d m_blocks=%lld n_blocks=%d",
                         layout, c.pair ? 256 : 128, c.bn, c.stages, c.ks, plan.ksplit, c.pair, c.wg, sms,
                         static_cast<long long>(c.pair ? pair_rows : m_blocks), (N + c.bn - 1) / c.bn);
}

const char *dg_status_string(dg_status_t status)
{
    switch (status) {
    case DG_OK: return "DG_OK";
    case DG_ERR_INVALID_ARG: return "DG_ERR_INVALID_ARG";
    case DG_ERR_UNSUPPORTED: return "DG_ERR_UNSUPPORTED";
    case DG_ERR_ALIGNMENT: return "DG_ERR_ALIGNMENT";
    case DG_ERR_CUDA: return "DG_ERR_CUDA";
    case DG_ERR_TIMEOUT: return "DG_ERR_TIMEOUT";
    case DG_ERR_BAD_GROUP_DATA: return "DG_ERR_BAD_GROUP_DATA";
    case DG_ERR_WORKSPACE_LIMIT: return "DG_ERR_WORKSPACE_LIMIT";
    case DG_ERR_BAD_SCALE: return "DG_ERR_BAD_SCALE";
    }
    return "DG_ERR_UNKNOWN";
}

}  // extern "C"

// ====================================================== no-allocation variant
//
// dg_fp8_gemm_nt_noalloc: the dense GEMM through the K-split kernel, with the
// split partials in a fixed array compiled into this library instead of a
// workspace obtained with cudaMalloc.  For callers that must not have device
// memory allocated behind their back: frameworks whose caching pool hands
// out all device memory (an outside allocation can fail or fragment that
// pool), and latency-critical loops where the device-wide synchronisation
// that cudaMalloc/cudaFree may cause is not acceptable.

namespace {

// Split count of the no-allocation path for an M x N x K problem on `sms`
// SMs: the planner's own when it splits this shape, else the largest of
// 16, 8, 4, 2 that gives every split the same number (at least two) of K
// blocks -- no split is left empty -- and whose cluster the device can
// schedule within the SM cap; then lowered (through the same rule, down to
// 1) until the partials fit the fixed scratch.  Returns 0 when even S = 1
// does not fit.
int noalloc_split(int M, int N, int K, int sms)
{
    const int num_kb = K / 128;
    const int64_t tiles = static_cast<int64_t>((M + 127) / 128) * ((N + kNoAllocBN - 1) / kNoAllocBN);
    const size_t per_split = static_cast<size_t>(tiles) * kNoAllocBN * dg::kBM * sizeof(float);
    auto usable = [&](int S) {
        if (S == 1)
            return true;
        const int kbps = (num_kb + S - 1) / S;
        if (kbps < 2 || (num_kb + kbps - 1) / kbps != S || S > sms)
            return false;
        return max_active_clusters(kTileChoices[4], S) > 0;
    };
    const Plan plan = choose_plan((M + 127) / 128, (M + 255) / 256, N, num_kb, sms, true);
    int S = (plan.c.split && plan.c.bn == kNoAllocBN) ? plan.ksplit : 16;
    while (S > 1 && (!usable(S) || per_split * S > kNoAllocScratchBytes))
        S /= 2;
    return per_split * S > kNoAllocScratchBytes ? 0 : S;
}
}  // namespace

// The fixed scratch.  Every GPU that loads this library holds it until the
// process exits.  Host code must not use this name as a device address (on
// the host it is only a stand-in symbol); the set-up below asks the runtime
// for the real address on each device.
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

namespace {
std::mutex g_noalloc_mutex;
float *g_noalloc_addr[kMaxDevices] = {};

// Once per device, with that device current: the device address of the
// fixed scratch.
dg_status_t noalloc_scratch_address(float **out)
{
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices)
        return DG_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_addr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
            (void)cudaGetLastError();
            return DG_ERR_CUDA;
        }
        g_noalloc_addr[dev] = static_cast<float *>(ptr);
    }
    *out = g_noalloc_addr[dev];
    return DG_OK;
}
}  // namespace

extern "C" dg_status_t dg_fp8_gemm_nt_noalloc(const void *A, const float *sA, const void *B,
                                               const float *sB, void *D, int M, int N, int K,
                                               cudaStream_t stream)
{
    if (M < 0)
        return DG_ERR_INVALID_ARG;
    dg_status_t st = check_common(A, sA, B, sB, D, N, K);
    if (st != DG_OK)
        return st;
    if (M == 0)
        return DG_OK;
    const int dev = current_device();
    const int sms = effective_sms(dev);
    if (sms <= 0)
        return DG_ERR_CUDA;

    // The K-split kernel's tile (BN = 144), split S ways (noalloc_split).
    constexpr int kBN = kNoAllocBN;
    const int S = noalloc_split(M, N, K, sms);
    if (S == 0)
        return DG_ERR_WORKSPACE_LIMIT;
    GemmParams p{};
    p.sA = sA;
    p.sB = sB;
    p.D = static_cast<__nv_bfloat16 *>(D);
    p.M = M;
    p.N = N;
    p.K = K;
    p.G = 1;
    p.sa_ld = dg_get_tma_aligned_size(M, 4);
    p.num_kb = K / 128;
    p.nbn = (N + 127) / 128;
    p.num_mb = (M + 127) / 128;
    p.num_nb = (N + kBN - 1) / kBN;
    p.raster = choose_raster(p.num_mb, dg::kBM, K);
    p.timeout_ns = g_timeout_ns.load();
    p.stamps = g_stamps.load();
    p.stall_injection = g_stall_injection.load();
    const int64_t tiles = static_cast<int64_t>(p.num_mb) * p.num_nb;
    const size_t per_split = static_cast<size_t>(tiles) * kBN * dg::kBM * sizeof(float);
    p.ksplit = S;
    p.kb_per_split = (p.num_kb + S - 1) / S;
    st = noalloc_scratch_address(&p.ws);
    if (st != DG_OK)
        return st;
    if (print_configs())
        std::fprintf(stderr, "[dg] dense (no-alloc) M=%d N=%d K=%d -> BN=%d ksplit=%d scratch=%zu B\n",
                     M, N, K, kBN, S, per_split * S);
    return launch_kernel<kBN, 3, 2, dg::kDense, true>(A, static_cast<uint64_t>(M), B,
                                                      static_cast<uint64_t>(N), p,
                                                      static_cast<int>(tiles * S), stream);
}
