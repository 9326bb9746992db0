/*
 * fg8_oracle.c -- plain CPU oracle for the fine-grained-scaled FP8 GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline leg of bench.py may load this code.  It shares no source,
 * header, table or helper with the CUDA library, and neither side includes
 * or links the other.
 *
 * What it computes (all accumulation in IEEE double):
 *
 *   D[m,n] = sum_kb ( sum_{k in kb} dec(A[m,k]) * dec(B[n,k]) )
 *                   * sfa[m,kb] * sfb[floor(n/128), kb]
 *
 * with 128-wide K blocks, E4M3 operands, one FP32 scale per 1x128 row block
 * of A and one per 128x128 block of B.  Sources:
 *   - fine-grained scaling "as proposed in DeepSeek-V3": chujupifa.com
 *     "机器之心报道" (DeepGEMM release report), opening summary; and
 *     deepseek.csdn.net "DeepGEMM：简洁、高效，用约300行CUDA代码重构AI计算的底层法则",
 *     section "什么是DeepGEMM呢？".
 *   - E4M3 = 4 exponent bits + 3 mantissa bits: ai.abqq.net
 *     "DeepSeek开源周第三天…开源项目DeepGEMM：FP8", section 3 "核心功能与特性".
 *   - two-level accumulation (each K block's partial sum is scaled and added
 *     into a wider accumulator): chujupifa.com report, opening summary
 *     ("两级累加（提升）机制"); ai.abqq.net, section 1 "架构优化".
 *   - normal, contiguous-grouped and masked-grouped layouts: game.3loumao.org
 *     explainer, section "03 DeepSeek是如何创新的？"; ai.abqq.net section 3.
 *   - column-major TMA-aligned scale layout and alignment helpers:
 *     deepseek.csdn.net page, section "实用工具".
 *
 * Readings where the pages are silent (the E4M3 variant is OCP E4M3FN: bias 7,
 * subnormals at e=0, S.1111.111 is NaN, no infinities, max 448; block size 128;
 * FP32 scales multiply the decoded code) are listed in the design notes of the
 * repository, together with the pins that check every function here.
 *
 * The code is deliberately naive: two table lookups and one multiply-add per
 * product, no blocking, no vectorisation, OpenMP only over independent output
 * elements.  Every product dec(a)*dec(b) has at most 8 significant bits and
 * magnitude in [2^-18, 448^2], so each 128-term block sum is exact in double;
 * each block contributes one rounding (times the scales) and one addition.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define FG8O_BLOCK 128

/* E4M3 (OCP "FN" variant) code -> real value, from the bit fields.
 * sign = bit 7, exponent = bits 6..3 (bias 7), mantissa = bits 2..0.
 * e == 0: subnormal (m/8) * 2^-6.  e == 15 && m == 7: NaN.  No infinities. */
static double e4m3_decode(unsigned code)
{
    unsigned s = (code >> 7) & 1u;
    unsigned e = (code >> 3) & 0xFu;
    unsigned m = code & 0x7u;
    double mag;
    if (e == 15u && m == 7u)
        return NAN;
    if (e == 0u)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -mag : mag;
}

static double g_table[256];
static int g_table_ready = 0;

static void build_table(void)
{
    if (g_table_ready)
        return;
    for (unsigned c = 0; c < 256; ++c)
        g_table[c] = e4m3_decode(c);
    g_table_ready = 1;
}

void fg8o_e4m3_table(double *out256)
{
    build_table();
    memcpy(out256, g_table, sizeof(g_table));
}

int fg8o_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* One output element of the definition above.
 *   arow : K codes of one A row
 *   sfa_row : KB scales of that row (row-major [.][KB])
 *   brow : K codes of one B row (output column n)
 *   sfb_row : KB scales of the 128-row B block that holds n */
static double dot_scaled(const uint8_t *arow, const float *sfa_row,
                         const uint8_t *brow, const float *sfb_row, int K)
{
    int KB = K / FG8O_BLOCK;
    double acc = 0.0;
    for (int kb = 0; kb < KB; ++kb) {
        double partial = 0.0;
        for (int k = kb * FG8O_BLOCK; k < (kb + 1) * FG8O_BLOCK; ++k)
            partial += g_table[arow[k]] * g_table[brow[k]];
        double scale = (double)sfa_row[kb] * (double)sfb_row[kb];
        acc += partial * scale;
    }
    return acc;
}

/* Normal GEMM D = A . B^T with fine-grained scales.
 *   A   [M][K] codes, row-major        sfa [M][KB] fp32, row-major
 *   B   [N][K] codes, row-major        sfb [ceil(N/128)][KB] fp32, row-major
 *   rows: list of n_rows row indices of D to compute (NULL: all M rows)
 *   D   [n_rows][N] doubles (row i holds D[rows[i], :])
 * Returns 0, or -1 on bad sizes. */
int fg8o_gemm_nt(const uint8_t *A, const float *sfa, const uint8_t *B,
                 const float *sfb, int M, int N, int K, const int *rows,
                 int n_rows, double *D, int threads)
{
    if (M < 0 || N < 0 || K <= 0 || K % FG8O_BLOCK != 0)
        return -1;
    if (rows == NULL)
        n_rows = M;
    build_table();
    const int KB = K / FG8O_BLOCK;
    const long long total = (long long)n_rows * N;
#pragma omp parallel for schedule(static) num_threads(threads > 0 ? threads : fg8o_num_threads())
    for (long long idx = 0; idx < total; ++idx) {
        int i = (int)(idx / N);
        int n = (int)(idx % N);
        int m = rows ? rows[i] : i;
        D[idx] = dot_scaled(A + (size_t)m * K, sfa + (size_t)m * KB,
                            B + (size_t)n * K, sfb + (size_t)(n / FG8O_BLOCK) * KB, K);
    }
    return 0;
}

/* Contiguous-grouped GEMM: expert segments concatenated along M.
 *   A [M_tot][K], sfa [M_tot][KB]
 *   B [G][N][K], sfb [G][ceil(N/128)][KB]
 *   m_indices [M_tot]: expert of each row, -1 (or out of range) = padding,
 *                      never computed or written
 *   rows / n_rows / D as for fg8o_gemm_nt; written[i] = 1 when row rows[i]
 *   belongs to an expert, 0 when it is padding (then D row i is untouched). */
int fg8o_m_grouped_contiguous(const uint8_t *A, const float *sfa,
                              const uint8_t *B, const float *sfb,
                              const int *m_indices, int M_tot, int N, int K,
                              int G, const int *rows, int n_rows, double *D,
                              uint8_t *written, int threads)
{
    if (M_tot < 0 || N < 0 || G <= 0 || K <= 0 || K % FG8O_BLOCK != 0)
        return -1;
    if (rows == NULL)
        n_rows = M_tot;
    build_table();
    const int KB = K / FG8O_BLOCK;
    const int NB = (N + FG8O_BLOCK - 1) / FG8O_BLOCK;
    for (int i = 0; i < n_rows; ++i) {
        int m = rows ? rows[i] : i;
        int e = m_indices[m];
        written[i] = (uint8_t)(e >= 0 && e < G);
    }
    const long long total = (long long)n_rows * N;
#pragma omp parallel for schedule(static) num_threads(threads > 0 ? threads : fg8o_num_threads())
    for (long long idx = 0; idx < total; ++idx) {
        int i = (int)(idx / N);
        int n = (int)(idx % N);
        if (!written[i])
            continue;
        int m = rows ? rows[i] : i;
        int e = m_indices[m];
        const uint8_t *Be = B + (size_t)e * N * K;
        const float *sfbe = sfb + (size_t)e * NB * KB;
        D[idx] = dot_scaled(A + (size_t)m * K, sfa + (size_t)m * KB,
                            Be + (size_t)n * K, sfbe + (size_t)(n / FG8O_BLOCK) * KB, K);
    }
    return 0;
}

/* Masked-grouped GEMM: G independent problems of M_max rows each.
 *   A [G][M_max][K], sfa [G][M_max][KB]
 *   B [G][N][K],     sfb [G][ceil(N/128)][KB]
 *   masked_m [G]: rows r < min(masked_m[g], M_max) of group g are computed;
 *                 the others are never written.
 *   rows: list of flat row ids g*M_max + r (NULL: all G*M_max rows)
 *   D [n_rows][N]; written[i] as for the contiguous case. */
int fg8o_m_grouped_masked(const uint8_t *A, const float *sfa, const uint8_t *B,
                          const float *sfb, const int *masked_m, int G,
                          int M_max, int N, int K, const int *rows, int n_rows,
                          double *D, uint8_t *written, int threads)
{
    if (G <= 0 || M_max < 0 || N < 0 || K <= 0 || K % FG8O_BLOCK != 0)
        return -1;
    if (rows == NULL)
        n_rows = G * M_max;
    build_table();
    const int KB = K / FG8O_BLOCK;
    const int NB = (N + FG8O_BLOCK - 1) / FG8O_BLOCK;
    for (int i = 0; i < n_rows; ++i) {
        int flat = rows ? rows[i] : i;
        int g = flat / (M_max > 0 ? M_max : 1);
        int r = flat - g * M_max;
        int lim = masked_m[g] < M_max ? masked_m[g] : M_max;
        written[i] = (uint8_t)(r < lim);
    }
    const long long total = (long long)n_rows * N;
#pragma omp parallel for schedule(static) num_threads(threads > 0 ? threads : fg8o_num_threads())
    for (long long idx = 0; idx < total; ++idx) {
        int i = (int)(idx / N);
        int n = (int)(idx % N);
        if (!written[i])
            continue;
        int flat = rows ? rows[i] : i;
        int g = flat / M_max;
        const uint8_t *Bg = B + (size_t)g * N * K;
        const float *sfbg = sfb + (size_t)g * NB * KB;
        D[idx] = dot_scaled(A + (size_t)flat * K, sfa + (size_t)flat * KB,
                            Bg + (size_t)n * K, sfbg + (size_t)(n / FG8O_BLOCK) * KB, K);
    }
    return 0;
}

/* Smallest n' >= n such that n' * elem_bytes is a multiple of 16 bytes (the
 * TMA stride rule).  The csdn page lists get_tma_aligned_size among the
 * utilities (section "实用工具") without its formula; this is the plainest
 * reading. */
long long fg8o_tma_aligned_size(long long n, long long elem_bytes)
{
    if (elem_bytes <= 0 || 16 % elem_bytes != 0)
        return -1;
    long long a = 16 / elem_bytes;
    return (n + a - 1) / a * a;
}

/* Scale layout transform ("column-major, TMA-aligned" scale tensor; csdn
 * page, section "实用工具", get_col_major_tma_aligned_tensor):
 *   in  [G][M][KB]   fp32 row-major (one scale per 1x128 block of A)
 *   out [G][KB][M_pad] with M_pad = fg8o_tma_aligned_size(M, 4);
 *   out[g][kb][m] = in[g][m][kb] for m < M, 0 for M <= m < M_pad. */
int fg8o_sfa_to_mn_major(const float *in, float *out, int G, int M, int KB)
{
    if (G < 0 || M < 0 || KB < 0)
        return -1;
    long long M_pad = fg8o_tma_aligned_size(M, 4);
    for (int g = 0; g < G; ++g)
        for (int kb = 0; kb < KB; ++kb)
            for (long long m = 0; m < M_pad; ++m)
                out[((size_t)g * KB + kb) * M_pad + m] =
                    m < M ? in[((size_t)g * M + m) * KB + kb] : 0.0f;
    return 0;
}

/* ---- quantiser (input preparation; the step before the GEMM) ----------- */

/* Round an fp32 value to the nearest E4M3 code, ties to even code (the codes
 * of one sign are monotone in magnitude, so an even code is an even
 * mantissa), after saturating to +-448.  Found by scanning every finite code:
 * slow and plain on purpose. */
static uint8_t e4m3_encode_rne(float xf)
{
    build_table();
    double x = (double)xf;
    if (x != x)
        return 0x7F;
    if (x > 448.0)
        x = 448.0;
    if (x < -448.0)
        x = -448.0;
    unsigned sign = x < 0.0 || (x == 0.0 && signbit(x)) ? 0x80u : 0u;
    double ax = fabs(x);
    unsigned best = 0;
    double best_err = INFINITY;
    for (unsigned c = 0; c <= 0x7E; ++c) {
        double err = fabs(g_table[c] - ax);
        if (err < best_err || (err == best_err && (c & 1u) == 0u)) {
            best = c;
            best_err = err;
        }
    }
    return (uint8_t)(sign | best);
}

uint8_t fg8o_e4m3_encode(float x) { return e4m3_encode_rne(x); }

/* Block quantiser: x [R][C] fp32 row-major, blocks of br rows x 128 columns
 * (br = 1 for activations, 128 for weights; the last blocks may be partial).
 * scale = max(amax, 1e-4) / 448 in fp32; q = E4M3_RNE(clamp(x / scale)) with
 * the division in fp32.  s has ceil(R/br) rows of ceil(C/128) scales. */
int fg8o_quantize_blocks(const float *x, int R, int C, int br, uint8_t *q,
                         float *s)
{
    if (R < 0 || C < 0 || br <= 0)
        return -1;
    int CB = (C + FG8O_BLOCK - 1) / FG8O_BLOCK;
    int RB = (R + br - 1) / br;
    for (int rb = 0; rb < RB; ++rb) {
        for (int cb = 0; cb < CB; ++cb) {
            int r0 = rb * br, r1 = r0 + br < R ? r0 + br : R;
            int c0 = cb * FG8O_BLOCK, c1 = c0 + FG8O_BLOCK < C ? c0 + FG8O_BLOCK : C;
            float amax = 0.0f;
            for (int r = r0; r < r1; ++r)
                for (int c = c0; c < c1; ++c) {
                    float a = fabsf(x[(size_t)r * C + c]);
                    if (a > amax)
                        amax = a;
                }
            float scale = (amax > 1e-4f ? amax : 1e-4f) / 448.0f;
            s[(size_t)rb * CB + cb] = scale;
            for (int r = r0; r < r1; ++r)
                for (int c = c0; c < c1; ++c) {
                    float v = x[(size_t)r * C + c] / scale;
                    q[(size_t)r * C + c] = e4m3_encode_rne(v);
                }
        }
    }
    return 0;
}
