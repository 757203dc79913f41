/*
 * CPU oracle for the FP8 (E4M3) NT GEMM with fine-grained scaling.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check
 * and the benchmark's CPU-baseline leg may load this code.  It shares no code,
 * header, table or constant with the CUDA library, and it never calls it.
 *
 * What is computed (the plain definition, in FP64):
 *
 *   D[m,n] = sum_{kb} ( sum_{k in block kb} dec(A[m,k]) * dec(B[n,k]) )
 *                     * sa[m,kb] * sb[n/128, kb]
 *
 * - Operand format: E4M3 FP8 bytes (DeepGEMM README, introduction: FP8 GEMM
 *   with fine-grained scaling "as proposed in DeepSeek-V3"; the hnwysp.cn
 *   DeepGEMM blog, section 4.1, gives E4M3's range of about +-448).
 * - NT layout: A is [M,K] and B is [N,K], both K-contiguous (DeepGEMM README,
 *   usage: only the NT format, non-transposed LHS and transposed RHS).
 * - Scale granularity: one FP32 scale per LHS row per 128-wide K block and one
 *   per 128x128 RHS block (DeepSeek-V3 fine-grained scaling as cited above).
 * - LHS scales are column-major with leading dimension ld_sa (DeepGEMM README,
 *   usage: the LHS scaling factors must be transposed to a TMA-aligned
 *   column-major layout).
 * - Accumulation: the pages ask for FP32 accumulation (hnwysp.cn blog, section
 *   4.3, and the DeepGEMM README's two-level "promotion" on CUDA cores); the
 *   oracle accumulates in FP64, which is at least as precise.
 *
 * Exactness: every E4M3 value is an integer multiple of 2^-9 of magnitude at
 * most 448, so each product is an integer multiple of 2^-18 below 2^36 * 2^-18
 * and a 128-term block sum is an integer multiple of 2^-18 below 2^43 * 2^-18;
 * FP64's 53-bit significand holds it exactly, whatever the summation order.
 * The only rounding is in the scaled sum over K blocks.
 *
 * Grouped forms (DeepGEMM README, grouped GEMMs: only the M axis is grouped,
 * experts share N and K):
 * - contiguous: row m uses expert m_indices[m]; rows marked -1 are padding and
 *   are not computed (left as NaN in the result).
 * - masked: group g computes its first masked_m[g] rows only; other rows are
 *   not computed (left as NaN).
 *
 * All functions return 0 on success, nonzero on a bad argument.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>

#define ORACLE_BLOCK 128

/* E4M3 decoding from the bit fields: sign (bit 7), exponent (bits 6..3, bias
 * 7), mantissa (bits 2..0).  Exponent 0 is subnormal: m * 2^-9.  Exponent 15
 * with mantissa 7 is NaN; there are no infinities, so 0x7E = 448 is the
 * largest finite value. */
static double e4m3_decode(uint8_t byte)
{
    int sign = byte >> 7;
    int exponent = (byte >> 3) & 0xF;
    int mantissa = byte & 0x7;
    double magnitude;
    if (exponent == 15 && mantissa == 7)
        return NAN;
    if (exponent == 0)
        magnitude = ldexp((double)mantissa, -9);
    else
        magnitude = ldexp(8.0 + mantissa, exponent - 10); /* (1 + m/8) 2^(e-7) */
    return sign ? -magnitude : magnitude;
}

void oracle_e4m3_table(double *table256)
{
    for (int i = 0; i < 256; ++i)
        table256[i] = e4m3_decode((uint8_t)i);
}

/* One output element of the dense definition.
 * a_row: the K bytes of row m of A; b_row: the K bytes of row n of B;
 * sa_col: &sa[m] so that sa_col[kb * ld_sa] is sa[m, kb];
 * sb_row: &sb[(n / 128) * nkb] so that sb_row[kb] is sb[n / 128, kb]. */
static double element(const double *dec, const uint8_t *a_row, const uint8_t *b_row,
                      const float *sa_col, long ld_sa, const float *sb_row, int K)
{
    int nkb = (K + ORACLE_BLOCK - 1) / ORACLE_BLOCK;
    double d = 0.0;
    for (int kb = 0; kb < nkb; ++kb) {
        int k0 = kb * ORACLE_BLOCK;
        int k1 = k0 + ORACLE_BLOCK < K ? k0 + ORACLE_BLOCK : K;
        double partial = 0.0;
        for (int k = k0; k < k1; ++k)
            partial += dec[a_row[k]] * dec[b_row[k]];
        d += partial * (double)sa_col[(long)kb * ld_sa] * (double)sb_row[kb];
    }
    return d;
}

static int check_dims(int M, int N, int K, long ld_sa)
{
    if (M < 0 || N < 0 || K <= 0 || ld_sa < M)
        return 1;
    return 0;
}

/* Dense: D[M*N] (row-major, FP64) for A[M,K], sa[nkb][ld_sa], B[N,K],
 * sb[ceil(N/128)][nkb]. */
int oracle_gemm_dense(const uint8_t *A, const float *sa, long ld_sa, const uint8_t *B,
                      const float *sb, int M, int N, int K, double *D)
{
    if (check_dims(M, N, K, ld_sa))
        return 1;
    double dec[256];
    oracle_e4m3_table(dec);
    int nkb = (K + ORACLE_BLOCK - 1) / ORACLE_BLOCK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n)
            D[(long)m * N + n] = element(dec, A + (long)m * K, B + (long)n * K, sa + m, ld_sa,
                                         sb + (long)(n / ORACLE_BLOCK) * nkb, K);
    return 0;
}

/* Dense, at listed positions only: D_out[i] = D[rows[i], cols[i]]. */
int oracle_gemm_dense_sampled(const uint8_t *A, const float *sa, long ld_sa, const uint8_t *B,
                              const float *sb, int M, int N, int K, const int *rows,
                              const int *cols, long count, double *D_out)
{
    if (check_dims(M, N, K, ld_sa))
        return 1;
    for (long i = 0; i < count; ++i)
        if (rows[i] < 0 || rows[i] >= M || cols[i] < 0 || cols[i] >= N)
            return 2;
    double dec[256];
    oracle_e4m3_table(dec);
    int nkb = (K + ORACLE_BLOCK - 1) / ORACLE_BLOCK;
#pragma omp parallel for schedule(static)
    for (long i = 0; i < count; ++i) {
        int m = rows[i], n = cols[i];
        D_out[i] = element(dec, A + (long)m * K, B + (long)n * K, sa + m, ld_sa,
                           sb + (long)(n / ORACLE_BLOCK) * nkb, K);
    }
    return 0;
}

/* Contiguous grouped: A[M_sum,K], sa[nkb][ld_sa], B[G][N][K], sb[G][nnb][nkb],
 * m_indices[M_sum].  Rows with m_indices == -1 are left as NaN. */
int oracle_gemm_contiguous(const uint8_t *A, const float *sa, long ld_sa, const uint8_t *B,
                           const float *sb, const int *m_indices, int num_groups, int M_sum,
                           int N, int K, double *D)
{
    if (check_dims(M_sum, N, K, ld_sa) || num_groups <= 0)
        return 1;
    for (int m = 0; m < M_sum; ++m)
        if (m_indices[m] < -1 || m_indices[m] >= num_groups)
            return 2;
    double dec[256];
    oracle_e4m3_table(dec);
    int nkb = (K + ORACLE_BLOCK - 1) / ORACLE_BLOCK;
    int nnb = (N + ORACLE_BLOCK - 1) / ORACLE_BLOCK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int m = 0; m < M_sum; ++m) {
        int e = m_indices[m];
        for (int n = 0; n < N; ++n) {
            if (e < 0) {
                D[(long)m * N + n] = NAN;
                continue;
            }
            const uint8_t *Be = B + (long)e * N * K;
            const float *sbe = sb + (long)e * nnb * nkb;
            D[(long)m * N + n] = element(dec, A + (long)m * K, Be + (long)n * K, sa + m, ld_sa,
                                         sbe + (long)(n / ORACLE_BLOCK) * nkb, K);
        }
    }
    return 0;
}

/* Contiguous grouped at listed positions; a padding row gives NaN. */
int oracle_gemm_contiguous_sampled(const uint8_t *A, const float *sa, long ld_sa,
                                   const uint8_t *B, const float *sb, const int *m_indices,
                                   int num_groups, int M_sum, int N, int K, const int *rows,
                                   const int *cols, long count, double *D_out)
{
    if (check_dims(M_sum, N, K, ld_sa) || num_groups <= 0)
        return 1;
    for (long i = 0; i < count; ++i)
        if (rows[i] < 0 || rows[i] >= M_sum || cols[i] < 0 || cols[i] >= N ||
            m_indices[rows[i]] < -1 || m_indices[rows[i]] >= num_groups)
            return 2;
    double dec[256];
    oracle_e4m3_table(dec);
    int nkb = (K + ORACLE_BLOCK - 1) / ORACLE_BLOCK;
    int nnb = (N + ORACLE_BLOCK - 1) / ORACLE_BLOCK;
#pragma omp parallel for schedule(static)
    for (long i = 0; i < count; ++i) {
        int m = rows[i], n = cols[i], e = m_indices[m];
        if (e < 0) {
            D_out[i] = NAN;
            continue;
        }
        D_out[i] = element(dec, A + (long)m * K, B + ((long)e * N + n) * K, sa + m, ld_sa,
                           sb + ((long)e * nnb + n / ORACLE_BLOCK) * nkb, K);
    }
    return 0;
}

/* Masked grouped: A[G][M_max][K], sa[G][nkb][ld_sa], B[G][N][K], sb[G][nnb][nkb],
 * masked_m[G].  D[G][M_max][N]; rows at or beyond masked_m[g] are left as NaN. */
int oracle_gemm_masked(const uint8_t *A, const float *sa, long ld_sa, const uint8_t *B,
                       const float *sb, const int *masked_m, int G, int M_max, int N, int K,
                       double *D)
{
    if (check_dims(M_max, N, K, ld_sa) || G <= 0)
        return 1;
    for (int g = 0; g < G; ++g)
        if (masked_m[g] < 0 || masked_m[g] > M_max)
            return 2;
    double dec[256];
    oracle_e4m3_table(dec);
    int nkb = (K + ORACLE_BLOCK - 1) / ORACLE_BLOCK;
    int nnb = (N + ORACLE_BLOCK - 1) / ORACLE_BLOCK;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int g = 0; g < G; ++g)
        for (int m = 0; m < M_max; ++m) {
            double *Drow = D + ((long)g * M_max + m) * N;
            if (m >= masked_m[g]) {
                for (int n = 0; n < N; ++n)
                    Drow[n] = NAN;
                continue;
            }
            const uint8_t *Ag = A + (long)g * M_max * K;
            const float *sag = sa + (long)g * nkb * ld_sa;
            const uint8_t *Bg = B + (long)g * N * K;
            const float *sbg = sb + (long)g * nnb * nkb;
            for (int n = 0; n < N; ++n)
                Drow[n] = element(dec, Ag + (long)m * K, Bg + (long)n * K, sag + m, ld_sa,
                                  sbg + (long)(n / ORACLE_BLOCK) * nkb, K);
        }
    return 0;
}

/* Masked grouped at listed (g, m, n) positions; masked-out rows give NaN. */
int oracle_gemm_masked_sampled(const uint8_t *A, const float *sa, long ld_sa, const uint8_t *B,
                               const float *sb, const int *masked_m, int G, int M_max, int N,
                               int K, const int *groups, const int *rows, const int *cols,
                               long count, double *D_out)
{
    if (check_dims(M_max, N, K, ld_sa) || G <= 0)
        return 1;
    for (long i = 0; i < count; ++i)
        if (groups[i] < 0 || groups[i] >= G || rows[i] < 0 || rows[i] >= M_max ||
            cols[i] < 0 || cols[i] >= N)
            return 2;
    double dec[256];
    oracle_e4m3_table(dec);
    int nkb = (K + ORACLE_BLOCK - 1) / ORACLE_BLOCK;
    int nnb = (N + ORACLE_BLOCK - 1) / ORACLE_BLOCK;
#pragma omp parallel for schedule(static)
    for (long i = 0; i < count; ++i) {
        int g = groups[i], m = rows[i], n = cols[i];
        if (m >= masked_m[g]) {
            D_out[i] = NAN;
            continue;
        }
        D_out[i] = element(dec, A + ((long)g * M_max + m) * K, B + ((long)g * N + n) * K,
                           sa + (long)g * nkb * ld_sa + m, ld_sa,
                           sb + ((long)g * nnb + n / ORACLE_BLOCK) * nkb, K);
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * 1x128 activation quantiser (the step before the GEMM: the DeepGEMM README,
 * usage, leaves the cast and the transposition of the LHS scales to a
 * preceding kernel; the DeepSeek-V3 recipe cited above fixes the 1x128 tile).
 *
 * Reading (the pages give no formula): per row m and 128-wide K block kb,
 *   amax = max |x[m,k]| over the block              (FP32, exact)
 *   s    = max(amax, 1e-4) / 448                    (FP32 division, RN)
 *   q    = E4M3( clamp(x / s, -448, 448) )          (FP32 division, RN;
 *          round to nearest E4M3 value, ties to the even mantissa)
 * so that x ~ dec(q) * s; s goes to sa[kb * ld_sa + m] (column-major).
 * Inputs must be finite.
 */

/* Nearest E4M3 byte to a finite float in [-448, 448], ties to the even
 * mantissa bit, by search over the decode table (no bit tricks). */
static uint8_t e4m3_encode_nearest(float y, const double *dec)
{
    double v = (double)y;
    uint8_t best = 0;
    double best_err = INFINITY;
    for (int code = 0; code < 256; ++code) {
        double d = dec[code];
        if (isnan(d))
            continue;
        /* zero is stored as +0 for a non-negative input and -0 otherwise */
        if (d == 0.0 && (code == 0x80) != (signbit(y) != 0))
            continue;
        double err = fabs(d - v);
        if (err < best_err || (err == best_err && (code & 1) == 0 && (best & 1) == 1)) {
            best = (uint8_t)code;
            best_err = err;
        }
    }
    return best;
}

int oracle_quantize_1x128(const float *x, int M, int K, uint8_t *q, float *sa, long ld_sa)
{
    if (M < 0 || K <= 0 || K % ORACLE_BLOCK != 0 || ld_sa < M)
        return 1;
    double dec[256];
    oracle_e4m3_table(dec);
    const int nkb = K / ORACLE_BLOCK;
    const float floor_amax = 1e-4f;
    const float e4m3_max = 448.0f;
#pragma omp parallel for schedule(static)
    for (int m = 0; m < M; ++m) {
        for (int kb = 0; kb < nkb; ++kb) {
            const float *xb = x + (long)m * K + (long)kb * ORACLE_BLOCK;
            float amax = 0.0f;
            for (int k = 0; k < ORACLE_BLOCK; ++k) {
                float a = fabsf(xb[k]);
                if (a > amax)
                    amax = a;
            }
            if (amax < floor_amax)
                amax = floor_amax;
            volatile float s = amax / e4m3_max; /* one FP32 rounding */
            for (int k = 0; k < ORACLE_BLOCK; ++k) {
                volatile float y = xb[k] / s;
                float yc = y;
                if (yc > e4m3_max)
                    yc = e4m3_max;
                if (yc < -e4m3_max)
                    yc = -e4m3_max;
                q[(long)m * K + (long)kb * ORACLE_BLOCK + k] = e4m3_encode_nearest(yc, dec);
            }
            sa[(long)kb * ld_sa + m] = s;
        }
    }
    return 0;
}
