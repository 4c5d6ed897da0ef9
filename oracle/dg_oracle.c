/*
 * dg_oracle.c -- plain, slow CPU oracle for the fine-grained-scaled FP8 GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link or call
 * this file: only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark use it.  It shares no code, header, table or helper with the CUDA
 * library.
 *
 * What it computes (one definition, written out directly):
 *
 *   D[m,n] = bf16_RNE( sum_kb  sA[m,kb] * sB[n/128,kb] * P_kb[m,n] )
 *   P_kb[m,n] = sum_{k=128kb}^{128kb+127} dec(A[m,k]) * dec(B[n,k])
 *
 * Sources:
 *  - "DeepGEMM: kernel FP8 GEMM sach va hieu qua nho scaling chi tiet"
 *    (vi.news.hada.io/topic?id=19459), section "Giao dien GEMM va rang buoc
 *    layout": the NT form D = C + A @ B.T with A row-major and B given N x K
 *    (the C term is absent here, i.e. C = 0).
 *  - "deepseek开源周第三天：DeepGEMM深度分析" (pxiaoer.blog), the FP8-training
 *    list: one scale per 1x128 activation block and per 128x128 weight block,
 *    and intermediate results kept in FP32-or-better between blocks; section
 *    "DeepGEMM介绍": two-level accumulation, the tensor-core partial of one
 *    block promoted into a wider accumulator.
 *  - DeepGEMM article (lqnn.cn/news/60274), section "DeepGEMM": fine-grained
 *    scaling with CUDA-core two-level accumulation.
 *  - Grouped layouts: hada.io page, section "Dense va Grouped GEMM"
 *    (contiguous: rows of all experts concatenated along M, each expert's
 *    segment aligned to the M block; masked: only the valid rows of each
 *    group are computed).
 *
 * Arithmetic: each 128-wide block sum is formed in double.  It is exact:
 * every e4m3 product is a multiple of 2^-18 with magnitude below 2^18, so a
 * sum of 128 of them needs at most 43 significant bits.  The scale product
 * and the outer sum are also taken in double.  The result is rounded once,
 * from double straight to bf16 (round to nearest, ties to even), so there is
 * no double rounding through float.
 *
 * e4m3 is read as the "fn" variant (bias 7, no infinities, S.1111.111 = NaN,
 * largest finite value 448), the reading that matches the 448 in the
 * amax/448 scale rule.
 *
 * Scale layouts taken here are the LOGICAL ones:
 *   sA: [rows][K/128]   (one fp32 per 1x128 block of A)
 *   sB: [ceil(N/128)][K/128]   (one fp32 per 128x128 block of B)
 * and, for grouped problems, one such array per group, groups outermost.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define DGO_BLOCK 128

/* ------------------------------------------------------------------ codecs */

/* e4m3fn code -> exact value.  Normal: (1 + m/8) * 2^(e-7); subnormal
 * (e == 0): (m/8) * 2^-6; code S.1111.111 is NaN. */
double dgo_e4m3_value(uint8_t code)
{
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return s ? -NAN : NAN;
    if (e == 0)
        v = ldexp((double)m, -9);          /* m/8 * 2^-6 */
    else
        v = ldexp((double)(8 + m), e - 10); /* (8+m)/8 * 2^(e-7) */
    return s ? -v : v;
}

static double g_lut[256];
static int g_lut_ready = 0;

static void dgo_init_lut(void)
{
    if (g_lut_ready)
        return;
    for (int c = 0; c < 256; ++c)
        g_lut[c] = dgo_e4m3_value((uint8_t)c);
    g_lut_ready = 1;
}

void dgo_decode_e4m3(const uint8_t *in, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = dgo_e4m3_value(in[i]);
}

/* double -> bf16 bits, round to nearest even, one rounding step.
 * bf16 has 8 significant bits; normal exponents -126..127, subnormal
 * quantum 2^-133; values at or above (2^8 - 1/2) * 2^120 overflow to inf. */
uint16_t dgo_bf16_from_double(double x)
{
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    if (isnan(x))
        return (uint16_t)(sign | 0x7FC0u);
    double a = fabs(x);
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0)
        return sign;
    int e2;
    (void)frexp(a, &e2);          /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;               /* a in [2^E, 2^(E+1)) */
    int qexp = (E < -126) ? -133 : E - 7;
    double r = ldexp(a, -qexp);   /* exact: power-of-two scaling */
    double nq = nearbyint(r);     /* default rounding mode: ties to even */
    double v = ldexp(nq, qexp);
    if (v >= ldexp(1.0, 128))
        return (uint16_t)(sign | 0x7F80u);
    float f = (float)v;           /* exact: v is a bf16 value */
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    return (uint16_t)(sign | (uint16_t)((bits >> 16) & 0x7FFFu));
}

void dgo_bf16_round(const double *in, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = dgo_bf16_from_double(in[i]);
}

/* ------------------------------------------------------------ one element */

/* The definition for a single output element.  a_row: K codes of A's row;
 * b_row: K codes of B's row n; sa_row: K/128 scales of A's row;
 * sb_row: K/128 scales of B's 128-row block that holds n. */
static double dgo_element(const uint8_t *a_row, const float *sa_row,
                          const uint8_t *b_row, const float *sb_row, int K)
{
    int nkb = K / DGO_BLOCK;
    double acc = 0.0;
    for (int kb = 0; kb < nkb; ++kb) {
        double partial = 0.0;
        for (int k = kb * DGO_BLOCK; k < (kb + 1) * DGO_BLOCK; ++k)
            partial += g_lut[a_row[k]] * g_lut[b_row[k]];
        double scale = (double)sa_row[kb] * (double)sb_row[kb];
        acc += scale * partial;
    }
    return acc;
}

static int dgo_check_dims(int M, int N, int K)
{
    if (M < 0 || N <= 0 || K <= 0 || K % DGO_BLOCK != 0)
        return -1;
    return 0;
}

/* ------------------------------------------------------------------- dense */

/* Dense NT.  A: [M][K] codes, B: [N][K] codes, sA: [M][K/128],
 * sB: [ceil(N/128)][K/128].  D64 (may be NULL): [M][N] unrounded result;
 * D16 (may be NULL): [M][N] bf16 bits.  Returns 0, or -1 on bad sizes. */
int dgo_gemm_nt(const uint8_t *A, const float *sA, const uint8_t *B,
                const float *sB, int M, int N, int K, double *D64,
                uint16_t *D16)
{
    if (dgo_check_dims(M, N, K))
        return -1;
    dgo_init_lut();
    int nkb = K / DGO_BLOCK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int m = 0; m < M; ++m) {
        for (int n = 0; n < N; ++n) {
            double v = dgo_element(A + (int64_t)m * K, sA + (int64_t)m * nkb,
                                   B + (int64_t)n * K,
                                   sB + (int64_t)(n / DGO_BLOCK) * nkb, K);
            if (D64)
                D64[(int64_t)m * N + n] = v;
            if (D16)
                D16[(int64_t)m * N + n] = dgo_bf16_from_double(v);
        }
    }
    return 0;
}

/* Dense NT with an accumulator: D = C + A.B^T, the "D = C + A @ B" form of
 * the hada.io page (section "Giao dien GEMM va rang buoc layout", where
 * fp8_gemm_nt computes D = C + A @ B.T).  The page gives C no type; here C
 * and D are fp32 [M][N] (the reading for accumulating into an fp32 buffer,
 * C may be the buffer D itself).  C[m,n] plus the exact double result of
 * dgo_gemm_nt is rounded once from double to fp32 (round to nearest even,
 * the C conversion under the default rounding mode). */
int dgo_gemm_nt_acc(const uint8_t *A, const float *sA, const uint8_t *B,
                    const float *sB, const float *C, int M, int N, int K,
                    double *D64, float *D32)
{
    if (dgo_check_dims(M, N, K) || !C)
        return -1;
    dgo_init_lut();
    int nkb = K / DGO_BLOCK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int m = 0; m < M; ++m) {
        for (int n = 0; n < N; ++n) {
            double v = (double)C[(int64_t)m * N + n] +
                       dgo_element(A + (int64_t)m * K, sA + (int64_t)m * nkb,
                                   B + (int64_t)n * K,
                                   sB + (int64_t)(n / DGO_BLOCK) * nkb, K);
            if (D64)
                D64[(int64_t)m * N + n] = v;
            if (D32)
                D32[(int64_t)m * N + n] = (float)v;
        }
    }
    return 0;
}

/* dgo_gemm_nt_acc at selected (row, col) pairs; C is the whole [M][N]
 * accumulator. */
int dgo_gemm_nt_acc_sampled(const uint8_t *A, const float *sA, const uint8_t *B,
                            const float *sB, const float *C, int M, int N, int K,
                            const int64_t *rows, const int64_t *cols, int64_t count,
                            double *out64, float *out32)
{
    if (dgo_check_dims(M, N, K) || !C)
        return -1;
    dgo_init_lut();
    int nkb = K / DGO_BLOCK;
    for (int64_t i = 0; i < count; ++i)
        if (rows[i] < 0 || rows[i] >= M || cols[i] < 0 || cols[i] >= N)
            return -1;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = rows[i], n = cols[i];
        double v = (double)C[m * N + n] +
                   dgo_element(A + m * K, sA + m * nkb, B + n * K,
                               sB + (n / DGO_BLOCK) * nkb, K);
        if (out64)
            out64[i] = v;
        if (out32)
            out32[i] = (float)v;
    }
    return 0;
}

/* K-grouped TN GEMM (the weight gradient of MoE experts): the hada.io
 * page, section "Dense va Grouped GEMM", names a grouping along the K axis
 * for MoE weight backward, with M and N fixed (k_grouped_fp8_gemm_tn_
 * contiguous).  Group g owns K rows [off[g], off[g+1]) (multiples of 128) of
 * A [K][M] and B [K][N], both stored MN-major (the TN layout), and
 *
 *   D_g[m,n] = sum_{kb in g} sA[kb,m] * sB[kb,n] * sum_{k in kb} dec(A[k,m]) * dec(B[k,n])
 *
 * with one fp32 scale per 128 rows of K and per column for both operands
 * (sA [K/128][M], sB [K/128][N]: the scale granularity runs along the
 * contraction, as the per-block promotion needs).  D is [G][M][N]; the sum
 * is formed in double (block sums exact, as in dgo_gemm_nt) and rounded
 * once to fp32.  An empty group gives zeros.  Returns -1 for bad offsets. */
int dgo_k_grouped_tn(const uint8_t *A, const float *sA, const uint8_t *B,
                     const float *sB, const int32_t *off, int G, int M, int N,
                     int K, double *D64, float *D32)
{
    if (G <= 0 || M <= 0 || N <= 0 || K < 0 || K % DGO_BLOCK || off[0] != 0 || off[G] != K)
        return -1;
    for (int g = 0; g < G; ++g)
        if (off[g + 1] < off[g] || off[g] % DGO_BLOCK)
            return -1;
    dgo_init_lut();
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int g = 0; g < G; ++g) {
        for (int m = 0; m < M; ++m) {
            for (int n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int kb = off[g] / DGO_BLOCK; kb < off[g + 1] / DGO_BLOCK; ++kb) {
                    double partial = 0.0;
                    for (int k = kb * DGO_BLOCK; k < (kb + 1) * DGO_BLOCK; ++k)
                        partial += g_lut[A[(int64_t)k * M + m]] * g_lut[B[(int64_t)k * N + n]];
                    acc += (double)sA[(int64_t)kb * M + m] * (double)sB[(int64_t)kb * N + n] * partial;
                }
                const int64_t o = ((int64_t)g * M + m) * N + n;
                if (D64)
                    D64[o] = acc;
                if (D32)
                    D32[o] = (float)acc;
            }
        }
    }
    return 0;
}

/* Dense NT at selected (row, col) pairs only, for problems too large to
 * compute whole.  Same layouts as dgo_gemm_nt. */
int dgo_gemm_nt_sampled(const uint8_t *A, const float *sA, const uint8_t *B,
                        const float *sB, int M, int N, int K,
                        const int64_t *rows, const int64_t *cols, int64_t count,
                        double *out64, uint16_t *out16)
{
    if (dgo_check_dims(M, N, K))
        return -1;
    dgo_init_lut();
    int nkb = K / DGO_BLOCK;
    for (int64_t i = 0; i < count; ++i)
        if (rows[i] < 0 || rows[i] >= M || cols[i] < 0 || cols[i] >= N)
            return -1;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = rows[i], n = cols[i];
        double v = dgo_element(A + m * K, sA + m * nkb, B + n * K,
                               sB + (n / DGO_BLOCK) * nkb, K);
        if (out64)
            out64[i] = v;
        if (out16)
            out16[i] = dgo_bf16_from_double(v);
    }
    return 0;
}

/* --------------------------------------------------- contiguous grouped */

/* Contiguous grouped layout: rows of all groups concatenated along M, each
 * group's segment starting on a multiple of DGO_BLOCK rows (the segments are
 * aligned to the M block), so every aligned block of DGO_BLOCK rows belongs
 * to the one group named by its first row.  Row m is written, with B_g and
 * sB_g, when g = m_indices[m] lies in [0, G) and equals the index of the
 * first row of its block.  Every other row is not written: padding rows
 * (negative index), the rows of a block whose first row is padding or out of
 * range, and rows whose index disagrees with their block's first row (input
 * that breaks the alignment rule; see dgo_check_contiguous_alignment).
 * A: [M_total][K], sA: [M_total][K/128], B: [G][N][K],
 * sB: [G][ceil(N/128)][K/128], D: [M_total][N]. */
int dgo_grouped_contiguous(const uint8_t *A, const float *sA, const uint8_t *B,
                           const float *sB, const int32_t *m_indices,
                           int M_total, int N, int K, int G, double *D64,
                           uint16_t *D16)
{
    if (dgo_check_dims(M_total, N, K) || G <= 0)
        return -1;
    dgo_init_lut();
    int nkb = K / DGO_BLOCK;
    int64_t nbn = (N + DGO_BLOCK - 1) / DGO_BLOCK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int m = 0; m < M_total; ++m) {
        int g = m_indices[m];
        if (g < 0 || g >= G || g != m_indices[(m / DGO_BLOCK) * DGO_BLOCK])
            continue;
        const uint8_t *Bg = B + (int64_t)g * N * K;
        const float *sBg = sB + (int64_t)g * nbn * nkb;
        for (int n = 0; n < N; ++n) {
            double v = dgo_element(A + (int64_t)m * K, sA + (int64_t)m * nkb,
                                   Bg + (int64_t)n * K,
                                   sBg + (int64_t)(n / DGO_BLOCK) * nkb, K);
            if (D64)
                D64[(int64_t)m * N + n] = v;
            if (D16)
                D16[(int64_t)m * N + n] = dgo_bf16_from_double(v);
        }
    }
    return 0;
}

/* Checks the contiguous layout's alignment rule: each expert's segment
 * starts on a multiple of `align` rows, so every aligned block carries at most
 * one group index, on its first row, the other rows carrying that index or a
 * padding tag (negative).  Returns the first offending row, or -1. */
int64_t dgo_check_contiguous_alignment(const int32_t *m_indices, int M_total,
                                       int align)
{
    for (int m = 0; m < M_total; ++m) {
        int32_t first = m_indices[(m / align) * align];
        if (m_indices[m] >= 0 && m_indices[m] != first)
            return m;
    }
    return -1;
}

/* ------------------------------------------------------- masked grouped */

/* Masked grouped layout: group g owns rows [0, max_m) of its slab; only rows
 * below min(masked_m[g], max_m) are computed, the others are not written.
 * A: [G][max_m][K], sA: [G][max_m][K/128], B: [G][N][K],
 * sB: [G][ceil(N/128)][K/128], D: [G][max_m][N]. */
int dgo_grouped_masked(const uint8_t *A, const float *sA, const uint8_t *B,
                       const float *sB, const int32_t *masked_m, int G,
                       int max_m, int N, int K, double *D64, uint16_t *D16)
{
    if (dgo_check_dims(max_m, N, K) || G <= 0)
        return -1;
    dgo_init_lut();
    int nkb = K / DGO_BLOCK;
    int64_t nbn = (N + DGO_BLOCK - 1) / DGO_BLOCK;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int g = 0; g < G; ++g) {
        for (int m = 0; m < max_m; ++m) {
            int valid = masked_m[g] < max_m ? masked_m[g] : max_m;
            if (m >= valid)
                continue;
            int64_t row = (int64_t)g * max_m + m;
            const uint8_t *Bg = B + (int64_t)g * N * K;
            const float *sBg = sB + (int64_t)g * nbn * nkb;
            for (int n = 0; n < N; ++n) {
                double v = dgo_element(A + row * K, sA + row * nkb,
                                       Bg + (int64_t)n * K,
                                       sBg + (int64_t)(n / DGO_BLOCK) * nkb, K);
                if (D64)
                    D64[row * N + n] = v;
                if (D16)
                    D16[row * N + n] = dgo_bf16_from_double(v);
            }
        }
    }
    return 0;
}

/* ------------------------------------------- fp32 promotion emulation */

/* Analysis aid, not a reference: the same sum with each block partial
 * rounded to float, the scale product taken in float and the promotion done
 * as a float fused multiply-add in block order -- what any fp32 promotion
 * does at best.  Used to measure how many elements of a large problem the
 * element-wise tolerance would reject even for an exact tensor-core partial.
 * Output: float values at the selected (row, col) pairs. */
int dgo_gemm_nt_fp32_promotion_sampled(const uint8_t *A, const float *sA,
                                       const uint8_t *B, const float *sB,
                                       int M, int N, int K, const int64_t *rows,
                                       const int64_t *cols, int64_t count,
                                       float *out32)
{
    if (dgo_check_dims(M, N, K))
        return -1;
    dgo_init_lut();
    int nkb = K / DGO_BLOCK;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = rows[i], n = cols[i];
        const uint8_t *a_row = A + m * K, *b_row = B + n * K;
        const float *sa_row = sA + m * nkb, *sb_row = sB + (n / DGO_BLOCK) * nkb;
        float acc = 0.0f;
        for (int kb = 0; kb < nkb; ++kb) {
            double partial = 0.0;
            for (int k = kb * DGO_BLOCK; k < (kb + 1) * DGO_BLOCK; ++k)
                partial += g_lut[a_row[k]] * g_lut[b_row[k]];
            float scale = sa_row[kb] * sb_row[kb];
            acc = fmaf((float)partial, scale, acc);
        }
        out32[i] = acc;
    }
    return 0;
}

int dgo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------- UE8M0 scales
 *
 * The block-scaled mode of the SM100 path takes its scales as UE8M0 (an
 * unsigned 8-bit biased exponent e, value 2^(e-127), e = 255 is NaN), four
 * of them packed into one 32-bit integer, in a transposed (MN-major) layout
 * (hada.io page, section "Giao dien GEMM va rang buoc layout": the SM100
 * scaling factors are packed UE8M0, four to an int, and the LHS scales are
 * TMA-aligned and transposed).
 *
 * Readings where the pages are silent:
 *  - byte j (bits 8j .. 8j+7) of the integer for row r and group g holds the
 *    scale of K block 4g + j; bytes past the last K block hold 127 (value 1);
 *  - the packed array is [ceil(nkb/4)][rows] (MN-major);
 *  - a UE8M0 quantiser picks, per block, the smallest power of two s with
 *    amax / s <= 448, i.e. s = 2^ceil(log2(amax / 448)), and the data is
 *    quantised with that s.
 * The GEMM itself is unchanged: with the scales decoded, dgo_gemm_nt and the
 * grouped forms above compute the block-scaled result.
 */

/* UE8M0 code -> value: 2^(e-127); e = 255 is NaN. */
double dgo_ue8m0_value(uint8_t e)
{
    if (e == 255)
        return NAN;
    return ldexp(1.0, (int)e - 127);
}

/* Exact encoding: s must be a power of two in [2^-127, 2^127]; returns its
 * code, or -1 for anything else (zero, negative, not a power of two, out of
 * range, inf, NaN). */
int dgo_ue8m0_from_scale(double s)
{
    if (!(s > 0.0) || isinf(s))
        return -1;
    int ex;
    double m = frexp(s, &ex); /* s = m * 2^ex, 0.5 <= m < 1 */
    if (m != 0.5)
        return -1;
    int e = ex - 1 + 127;
    if (e < 0 || e > 254)
        return -1;
    return e;
}

/* The smallest power of two >= x, for finite x > 0. */
double dgo_ue8m0_ceil_pow2(double x)
{
    int ex;
    double m = frexp(x, &ex);
    return m == 0.5 ? x : ldexp(1.0, ex);
}

/* s: [rows][nkb] fp32 scales (powers of two) -> out: [ceil(nkb/4)][rows]
 * packed codes.  Returns 1 (and leaves out partly written) if a scale is not
 * representable. */
int dgo_pack_ue8m0(const float *s, int rows, int nkb, int32_t *out)
{
    if (rows < 0 || nkb < 1)
        return 1;
    int ngroups = (nkb + 3) / 4;
    for (int g = 0; g < ngroups; ++g) {
        for (int r = 0; r < rows; ++r) {
            uint32_t word = 0;
            for (int j = 0; j < 4; ++j) {
                int kb = 4 * g + j;
                int code = 127;
                if (kb < nkb) {
                    code = dgo_ue8m0_from_scale((double)s[(int64_t)r * nkb + kb]);
                    if (code < 0)
                        return 1;
                }
                word |= (uint32_t)code << (8 * j);
            }
            out[(int64_t)g * rows + r] = (int32_t)word;
        }
    }
    return 0;
}

/* Inverse of dgo_pack_ue8m0: in [ceil(nkb/4)][rows] -> s [rows][nkb]. */
int dgo_unpack_ue8m0(const int32_t *in, int rows, int nkb, float *s)
{
    if (rows < 0 || nkb < 1)
        return 1;
    for (int r = 0; r < rows; ++r) {
        for (int kb = 0; kb < nkb; ++kb) {
            uint32_t word = (uint32_t)in[(int64_t)(kb / 4) * rows + r];
            uint8_t code = (uint8_t)((word >> (8 * (kb % 4))) & 0xFFu);
            s[(int64_t)r * nkb + kb] = (float)dgo_ue8m0_value(code);
        }
    }
    return 0;
}
