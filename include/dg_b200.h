/*
 * dg_b200.h -- C ABI of the B200 (sm_100a) fine-grained-scaled FP8 GEMM.
 *
 * One operation, three layouts:
 *
 *   D[m,n] = bf16( sum_kb sA[m,kb] * sB[n/128,kb] * sum_{k in block kb} A[m,k]*B[n,k] )
 *
 * A and B are FP8 e4m3 ("fn": bias 7, max 448, no infinities), both K-major
 * (the "NT" form D = A @ B.T).  There is one fp32 scale per 1x128 block of A
 * and one per 128x128 block of B.  Each 128-wide K block is contracted on the
 * tensor cores and its partial is then promoted into an fp32 accumulator on
 * the CUDA cores as acc += (sA*sB) * partial.  D is bf16, rounded to nearest
 * even once at the end.  A separately declared UE8M0 mode (the *_ue8m0 calls
 * below) takes power-of-two scales packed four to an int32 and lets the
 * tensor core apply them (block-scaled MMA, fp32 accumulation in TMEM).
 *
 * Sources (the DeepGEMM pages):
 *  - "DeepGEMM: kernel FP8 GEMM sach va hieu qua nho scaling chi tiet"
 *    (vi.news.hada.io/topic?id=19459):
 *      section "Giao dien GEMM va rang buoc layout" -- D = C + A @ B.T for the
 *      NT layout (C is absent here: D is overwritten); the LHS scale must be
 *      TMA-aligned and transposed; fp32 scales on the Hopper path;
 *      section "Dense va Grouped GEMM" -- contiguous grouping along M with
 *      each expert segment aligned to the M block; masked grouping for
 *      CUDA-graph decode, computing only the valid rows;
 *      section "Tien ich va bien moi truong" -- set/get_num_sms,
 *      get_mk_alignment_for_contiguous_layout, get_tma_aligned_size.
 *  - DeepGEMM article (lqnn.cn/news/60274), section "DeepGEMM": fine-grained
 *    scaling with two-level accumulation on the CUDA cores.
 *  - "deepseek开源周第三天：DeepGEMM深度分析" (pxiaoer.blog): 1x128 activation
 *    and 128x128 weight scale blocks.
 *
 * Conventions for every GEMM entry point:
 *  - All tensor pointers are DEVICE pointers on the current device, owned by
 *    the caller.  The library keeps no reference after the call returns.
 *  - Calls are asynchronous on `stream` (0 = legacy default stream).
 *  - Host-side validation runs first; on any failure the call returns a
 *    non-zero status and launches nothing.
 *  - The group metadata (m_indices, masked_m) is read only on the device, so
 *    the calls never synchronise with the host and can be captured in a CUDA
 *    graph after a first call on the device (which loads the module).
 *  - Problems found on the device (bad group data, a pipeline wait that ran
 *    past its time limit) never trap: the kernel records a code in a device
 *    status word, leaves the affected rows untouched and returns.  Read and
 *    clear it with dg_get_device_status().
 *  - Device memory: the persistent paths allocate nothing.  For dense shapes
 *    with too few output tiles to fill the GPU (decode shapes), the library
 *    splits each tile's K range over a cluster of 2..16 CTAs whose fp32
 *    partial tiles meet in a library-owned workspace (tiles x splits x
 *    BN x 128 floats; 8.6 MB for M=128, N=2112, K=7168).  It is allocated on
 *    the first such call on a device, grown when a larger one is needed and
 *    kept until exit -- so make that first call before any stream capture.
 *    Calls that take this path on one device share the workspace: they must
 *    not overlap on the GPU (issue them on one stream).
 *  - Layout constraints: K >= 128 and K % 128 == 0; N >= 16 and N % 16 == 0;
 *    A, B, D and sA 16-byte aligned; sB and the metadata 4-byte aligned.
 *  - Row-major, packed (no leading-dimension arguments).
 */
#ifndef DG_B200_H
#define DG_B200_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DG_OK = 0,
    DG_ERR_INVALID_ARG = 1,    /* null pointer, bad size or count           */
    DG_ERR_UNSUPPORTED = 2,    /* shape outside the layout constraints       */
    DG_ERR_ALIGNMENT = 3,      /* pointer not aligned as required            */
    DG_ERR_CUDA = 4,           /* a CUDA runtime or driver call failed       */
    DG_ERR_TIMEOUT = 5,        /* device: a pipeline wait ran out of time    */
    DG_ERR_BAD_GROUP_DATA = 6, /* device: m_indices / masked_m out of range  */
    DG_ERR_WORKSPACE_LIMIT = 7, /* problem too large for the fixed scratch of
                                   dg_fp8_gemm_nt_noalloc                    */
    DG_ERR_BAD_SCALE = 8        /* device: dg_transform_sf_ue8m0 met a scale
                                   that is not a UE8M0 power of two          */
} dg_status_t;

/*
 * Dense NT GEMM.
 *   A  : [M][K]            e4m3 codes, row-major (K-major)
 *   sA : [K/128][M_pad]    fp32, transposed and TMA-aligned:
 *                          M_pad = dg_get_tma_aligned_size(M, 4); element
 *                          (m, kb) at sA[kb * M_pad + m]; pad entries unread
 *   B  : [N][K]            e4m3 codes, row-major (K-major)
 *   sB : [ceil(N/128)][K/128] fp32, element (n/128, kb)
 *   D  : [M][N]            bf16, written whole
 * M == 0 is a no-op returning DG_OK.
 */
dg_status_t dg_fp8_gemm_nt(const void *A, const float *sA, const void *B,
                           const float *sB, void *D, int M, int N, int K,
                           cudaStream_t stream);

/*
 * The other three operand layouts of the dense GEMM (hada.io page, section
 * "Giao dien GEMM va rang buoc layout": the SM100 implementation supports
 * the NT, TN, NN and TT memory layouts).  Read as D = op(A) @ op(B) with
 * row-major storage, the letter n for an operand stored in its logical
 * shape (A as [M][K], B as [K][N]) and t for one stored transposed (A as
 * [K][M], B as [N][K]); dg_fp8_gemm_nt is the NT case:
 *   nn : A [M][K] (K-major),  B [K][N] (N-major)
 *   tn : A [K][M] (M-major),  B [K][N] (N-major)
 *   tt : A [K][M] (M-major),  B [N][K] (K-major)
 * sA, sB and D are as in dg_fp8_gemm_nt (sA [K/128][M_pad], sB
 * [ceil(N/128)][K/128], D [M][N] bf16).  An M-major A needs M % 16 == 0
 * (DG_ERR_UNSUPPORTED otherwise).  These layouts run on one-CTA tiles; an
 * N-major B uses 128- or 256-column tiles (whole 128-column boxes), and a
 * decode-shaped problem splits its K range over a cluster on 128-column
 * tiles (the library-owned split workspace of dg_fp8_gemm_nt, same rules).
 */
dg_status_t dg_fp8_gemm_nn(const void *A, const float *sA, const void *B,
                           const float *sB, void *D, int M, int N, int K,
                           cudaStream_t stream);
dg_status_t dg_fp8_gemm_tn(const void *A, const float *sA, const void *B,
                           const float *sB, void *D, int M, int N, int K,
                           cudaStream_t stream);
dg_status_t dg_fp8_gemm_tt(const void *A, const float *sA, const void *B,
                           const float *sB, void *D, int M, int N, int K,
                           cudaStream_t stream);

/*
 * K-grouped TN GEMM for MoE weight gradients (hada.io page, section "Dense
 * va Grouped GEMM": a grouping along the K axis, M and N fixed, named
 * k_grouped_fp8_gemm_tn_contiguous).  Group g owns K rows
 * [k_offsets[g], k_offsets[g+1]) of the shared K axis and
 *   D[g] = A[rows of g]^T @ B[rows of g],  D[g][m][n] fp32.
 *   A         : [K][M]  e4m3, M-major (M % 16 == 0)
 *   sA        : [K/128][M_pad] fp32, one scale per 128 rows of K and per m,
 *               M_pad = dg_get_tma_aligned_size(M, 4)
 *   B         : [K][N]  e4m3, N-major
 *   sB        : [K/128][N] fp32, one scale per 128 rows of K and per n
 *               (16-byte aligned)
 *   D         : [G][M][N] fp32, written whole (an empty group gives zeros)
 *   k_offsets : [G+1] int32 DEVICE array, k_offsets[0] = 0, non-decreasing
 *               multiples of 128, k_offsets[G] = K; read only on the device
 *               (a malformed group is computed as empty and flagged with
 *               DG_ERR_BAD_GROUP_DATA in the status word)
 * The pages give neither the scale granularity nor the output type: scales
 * per 128 K rows and per column of both operands (the granularity along the
 * contraction that per-block promotion needs) and an fp32 output are the
 * readings taken.  K == 0 zero-fills D.  Runs on one-CTA tiles of 128 or 256
 * columns.
 */
dg_status_t dg_fp8_k_grouped_gemm_tn_contiguous(const void *A, const float *sA, const void *B,
                                                const float *sB, float *D,
                                                const int32_t *k_offsets, int M, int N, int K,
                                                int num_groups, cudaStream_t stream);

/*
 * Dense NT GEMM with an accumulator: D = C + A @ B^T, the "D = C + A @ B"
 * form of the pages (hada.io page, section "Giao dien GEMM va rang buoc
 * layout": fp8_gemm_nt computes D = C + A @ B.T).  The pages give C no
 * type; here C and D are fp32 [M][N], row-major, 16-byte aligned, and C may
 * be D itself (in-place accumulation, D += A @ B^T).  A, sA, B, sB and the
 * layout rules are those of dg_fp8_gemm_nt; the fp32 promotion accumulator
 * of each output is added to C in fp32.  C == NULL returns
 * DG_ERR_INVALID_ARG.  M == 0 is a no-op returning DG_OK.
 */
dg_status_t dg_fp8_gemm_nt_acc(const void *A, const float *sA, const void *B,
                               const float *sB, const float *C, float *D, int M, int N,
                               int K, cudaStream_t stream);

/*
 * Contiguous-layout grouped GEMM (MoE, grouping along M; N and K shared).
 *   A         : [M_total][K]     e4m3; the rows of all groups concatenated
 *   sA        : [K/128][M_pad]   fp32, M_pad = dg_get_tma_aligned_size(M_total, 4)
 *   B         : [G][N][K]        e4m3, one weight matrix per group
 *   sB        : [G][ceil(N/128)][K/128] fp32
 *   D         : [M_total][N]     bf16
 *   m_indices : [M_total]        int32 group of each row; a negative value
 *                                marks a padding row
 * Each group's segment starts on a multiple of
 * dg_get_mk_alignment_for_contiguous_layout() rows (so M_total is a multiple
 * of it too).  Row m is computed with group m_indices[m]; padding rows are
 * left untouched.  A row whose index is >= G, or differs from the index of
 * the first row of its aligned block, is left untouched and raises
 * DG_ERR_BAD_GROUP_DATA in the device status word.
 */
dg_status_t dg_fp8_grouped_gemm_contiguous(const void *A, const float *sA,
                                           const void *B, const float *sB,
                                           void *D, const int32_t *m_indices,
                                           int M_total, int N, int K,
                                           int num_groups, cudaStream_t stream);

/*
 * Masked-layout grouped GEMM (MoE decode under CUDA graphs).
 *   A        : [G][max_m][K]     e4m3
 *   sA       : [G][K/128][max_m_pad] fp32, max_m_pad = dg_get_tma_aligned_size(max_m, 4)
 *   B        : [G][N][K]         e4m3
 *   sB       : [G][ceil(N/128)][K/128] fp32
 *   D        : [G][max_m][N]     bf16
 *   masked_m : [G]               int32, valid rows of each group (device)
 * Rows m < masked_m[g] of group g are computed; all other rows of D are left
 * untouched.  masked_m[g] > max_m is clamped to max_m and a negative value is
 * read as 0; both raise DG_ERR_BAD_GROUP_DATA in the device status word.
 * expected_m is a host-side hint of the typical masked_m used to pick the
 * tile shape (0 = use max_m); it never affects results.
 */
dg_status_t dg_fp8_grouped_gemm_masked(const void *A, const float *sA,
                                       const void *B, const float *sB, void *D,
                                       const int32_t *masked_m, int num_groups,
                                       int max_m, int N, int K, int expected_m,
                                       cudaStream_t stream);

/*
 * Dense NT GEMM that allocates no device memory (same arguments, layouts
 * and result as dg_fp8_gemm_nt).  The pages describe no such call.  It is
 * for callers that cannot let a library allocate device memory while they
 * run: frameworks that hand out all device memory from their own caching
 * pool (an outside cudaMalloc can fail once the pool holds the memory, or
 * fragment it), and latency-critical loops where the device-wide
 * synchronisation that cudaMalloc/cudaFree may cause is not acceptable.
 *
 * It runs the K-split kernel (128 x 144 tiles, each tile's K range split
 * over a cluster of S CTAs) with the fp32 partials in a fixed 32 MiB array
 * compiled into the library, which every GPU that loads the library holds
 * until the process exits.  S is the dense planner's split for the shape
 * when it splits, else the largest of 16, 8, 4, 2 that gives every split the
 * same number (at least two) of K blocks and whose cluster fits the SM cap
 * (dg_set_num_sms); it is lowered (by the same rule, down to 1) until the
 * partials, ceil(M/128) * ceil(N/144) * S * 73,728 bytes, fit.  A problem
 * that does not fit even with S = 1 is rejected with DG_ERR_WORKSPACE_LIMIT
 * before anything is launched.  dg_describe_config layout 6 reports S.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Every call uses the same array, and each call writes every part of it
 *    that it later reads, so nothing has to start at zero.  Two calls that
 *    overlap on the GPU (different streams, or a graph that runs them
 *    concurrently) race on the array: serialise them.
 *  - No cudaMalloc, cudaFree or other allocating routine is called.
 *  - If dg_get_device_status reports DG_ERR_TIMEOUT, D is undefined.
 */
dg_status_t dg_fp8_gemm_nt_noalloc(const void *A, const float *sA, const void *B,
                                   const float *sB, void *D, int M, int N, int K,
                                   cudaStream_t stream);

/*
 * UE8M0 block-scaled mode (a separately declared mode of the same GEMM).
 *
 * The SM100 path of the pages takes its scaling factors as packed UE8M0,
 * four to an int (hada.io page, section "Giao dien GEMM va rang buoc
 * layout").  UE8M0 is an unsigned 8-bit biased exponent: code e is the scale
 * 2^(e-127) (e = 255 is NaN), so every scale is a power of two.  The tensor
 * core then applies the scales itself (tcgen05.mma kind::mxf8f6f4 with block
 * scaling) and accumulates the whole K range in fp32:
 *
 *   D[m,n] = bf16( sum_kb 2^(ea[m,kb]-127) * 2^(eb[n/128,kb]-127)
 *                         * sum_{k in block kb} A[m,k]*B[n,k] )
 *
 * which is the fine-grained-scaled result for those (power-of-two) scales,
 * up to the order of the fp32 additions.  Quantising with power-of-two
 * scales (the smallest 2^k >= amax/448 per block) is the caller's part, as
 * the cast to FP8 is in the fp32-scale mode.
 *
 * Packed scale layouts (int32 words; byte j = bits 8j..8j+7 of the word for
 * K-block group g holds K block 4g+j, bytes past the last K block are
 * ignored; ng = ceil(K/512)):
 *   sfa : dense/contiguous [ng][M_pad], masked [G][ng][max_m_pad], with
 *         X_pad = dg_get_tma_aligned_size(X, 4) (transposed, TMA-aligned,
 *         16-byte aligned base); pad entries unread
 *   sfb : [G][ng][ceil(N/128)] (G = 1 for dense), one word per 128x128
 *         weight block, 4-byte aligned
 * dg_transform_sf_ue8m0 builds both from the fp32 scale layouts.  A, B, D,
 * m_indices, masked_m, the validation rules and the device status behaviour
 * are those of dg_fp8_gemm_nt, dg_fp8_grouped_gemm_contiguous and
 * dg_fp8_grouped_gemm_masked.  These calls run one-CTA tiles (128 x BN, BN
 * in {128, 160, 192, 224}) or CTA-pair tiles (256 x BN); a dense problem with
 * too few tiles to fill the GPU splits K over a cluster of CTAs and uses the
 * library-owned split workspace described above (same rules: make the first
 * such call before any stream capture, and do not overlap such calls on the
 * GPU).  Everything else allocates nothing.
 */
dg_status_t dg_fp8_gemm_nt_ue8m0(const void *A, const int32_t *sfa, const void *B,
                                 const int32_t *sfb, void *D, int M, int N, int K,
                                 cudaStream_t stream);
dg_status_t dg_fp8_grouped_gemm_contiguous_ue8m0(const void *A, const int32_t *sfa,
                                                 const void *B, const int32_t *sfb, void *D,
                                                 const int32_t *m_indices, int M_total, int N,
                                                 int K, int num_groups, cudaStream_t stream);
dg_status_t dg_fp8_grouped_gemm_masked_ue8m0(const void *A, const int32_t *sfa, const void *B,
                                             const int32_t *sfb, void *D,
                                             const int32_t *masked_m, int num_groups,
                                             int max_m, int N, int K, int expected_m,
                                             cudaStream_t stream);

/*
 * Packs fp32 scales into the UE8M0 words above (the pages'
 * transform_sf_into_required_layout, hada.io page, section "Tien ich va bien
 * moi truong", for the SM100 format).  K is the GEMM's K (nkb = K/128 scales
 * per row); batch is 1, or G for per-group scale arrays.
 *   mn_major = 1: sf [batch][nkb][rows_pad] (the LHS-scale layout, rows_pad =
 *                 dg_get_tma_aligned_size(rows, 4)) -> out [batch][ng][rows_pad]
 *   mn_major = 0: sf [batch][rows][nkb] (the weight-scale layout, rows =
 *                 ceil(N/128)) -> out [batch][ng][rows]
 * Each scale must be a power of two in [2^-127, 2^127] (an fp32 value with a
 * zero mantissa, or the subnormal 2^-127); its code is exact.  Any other
 * value is packed as 255 (NaN, so the GEMM result shows it) and raises
 * DG_ERR_BAD_SCALE in the device status word.  Pad rows and bytes past the
 * last K block become 127 (scale 1).  Device pointers, asynchronous on
 * `stream`; rows == 0 is a no-op.
 */
dg_status_t dg_transform_sf_ue8m0(const float *sf, int32_t *out, int rows, int K, int batch,
                                  int mn_major, cudaStream_t stream);

/* Row alignment of each group's segment in the contiguous layout (128). */
int dg_get_mk_alignment_for_contiguous_layout(void);

/* x rounded up so that x * elem_bytes is a multiple of 16 bytes (the TMA
 * alignment of the transposed LHS-scale rows).  elem_bytes must be 1, 2, 4,
 * 8 or 16; returns -1 otherwise or when x < 0. */
int dg_get_tma_aligned_size(int x, int elem_bytes);

/* Caps the number of SMs the persistent kernels use (0 = all SMs of the
 * current device).  Returns DG_ERR_INVALID_ARG for n < 0. */
dg_status_t dg_set_num_sms(int n);

/* SMs the next launch on the current device will use. */
int dg_get_num_sms(void);

/* Tile families the planner may choose from (process-wide; for tuning and
 * tests -- the default lets the cost model decide).  One-CTA tiles are
 * 128 rows on one SM; pair tiles are 256 rows on the two SMs of a cluster
 * sharing one tcgen05 cta_group::2 MMA.  Forcing pair tiles also lifts the
 * rule that they are used only when they fill every SM pair.  The K-split
 * decode path is a one-CTA family.  Returns DG_ERR_INVALID_ARG for any other
 * value.  (A tuning control of this library; the pages have no counterpart.) */
#define DG_TILES_AUTO 0
#define DG_TILES_ONE_CTA 1
#define DG_TILES_PAIR 2
dg_status_t dg_set_tile_family(int family);

/* Pins the planner's tile width (BLOCK_N) to n, one of the compiled widths
 * (112, 128, 144, 160, 192, 224, 256; 144 is the K-split decode tile), or 0
 * to let the cost model decide (the default; DG_FORCE_BLOCK_N sets the
 * initial value).  Process-wide, for tuning and tests: a call whose layout
 * and tile family have no tile of that width takes the first tile of its
 * table.  Returns DG_ERR_INVALID_ARG for any other n.  (A tuning control of
 * this library; the pages have no counterpart.) */
dg_status_t dg_set_block_n(int n);

/* Launch timing.  While `stamps` (a DEVICE array of two unsigned 64-bit
 * integers, 8-byte aligned) is set, every GEMM launch folds the %globaltimer
 * time (ns) at which its first CTA started into stamps[0] (atomic minimum)
 * and the time at which its last CTA ended into stamps[1] (atomic maximum):
 * the caller sets stamps[0] = UINT64_MAX and stamps[1] = 0 before the
 * launches it wants to span, and stamps[1] - stamps[0] is their duration on
 * the device, without launch latency.  NULL (the default) turns it off.
 * Process-wide; the cost is two atomics per CTA.  (A measurement hook of
 * this library; the pages have no counterpart.) */
dg_status_t dg_set_timing_stamps(unsigned long long *stamps);

/* Tensor maps (TMA descriptors) the library has encoded so far in this
 * process.  Each call looks its maps up in a cache keyed by buffer address,
 * shape, strides, box and swizzle, so a call repeated on the same buffers
 * encodes none and leaves this count unchanged. */
unsigned long long dg_get_tensor_map_encodes(void);

/* Device allocations (cudaMalloc) the library has made so far in this
 * process: the K-split workspace, allocated on first use per device and
 * grown when a larger one is needed.  dg_fp8_gemm_nt_noalloc never adds to
 * it. */
unsigned long long dg_get_device_allocations(void);

/* Time limit of each pipeline wait inside the kernels, in nanoseconds
 * (default 2e9).  A wait that runs past it makes the kernel record
 * DG_ERR_TIMEOUT, drain its in-flight copies and return.  The output of a
 * call that reported DG_ERR_TIMEOUT is undefined (the K-split paths write NaN
 * into the columns of a split that gave up).  0 restores the default. */
dg_status_t dg_set_wait_timeout_ns(uint64_t ns);

/* Test hook for the bounded-wait path (0 = off, the default).  While on,
 * the producer warp of CTA 0 of every GEMM launch issues no loads, so that
 * CTA's pipeline waits never complete: they run out after the limit of
 * dg_set_wait_timeout_ns, the kernel records DG_ERR_TIMEOUT and returns with
 * its copies drained and TMEM freed, and the results are garbage.  Nothing
 * faults or hangs; turn it off again before real work. */
dg_status_t dg_set_stall_injection(int enable);

/* Synchronises `stream`, then returns the device status word of the current
 * device (DG_OK if no kernel reported a problem) and clears it.  The word
 * also holds details; see dg_get_device_status_detail. */
dg_status_t dg_get_device_status(cudaStream_t stream);

/* Like dg_get_device_status but also returns the raw 32-bit word (code in
 * bits 0-7, role in bits 8-11, stage in bits 12-19, CTA in bits 20-31) and
 * does not clear it. */
dg_status_t dg_get_device_status_detail(cudaStream_t stream, uint32_t *word);

/* Describes the kernel configuration the library would launch for a problem
 * (layout 0 = dense, 1 = contiguous, 2 = masked, and 3, 4, 5 for the same
 * layouts in the UE8M0 block-scaled mode; 6 = dense through
 * dg_fp8_gemm_nt_noalloc, ksplit=0 when it does not fit its scratch; for
 * masked, M = expected_m and groups = G) into buf (NUL-terminated, truncated
 * to len).  Returns the number of characters it wanted to write, or -1 on
 * bad arguments. */
int dg_describe_config(int layout, int M, int N, int K, int groups, char *buf,
                       int len);

/* Human-readable name of a status code. */
const char *dg_status_string(dg_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* DG_B200_H */
