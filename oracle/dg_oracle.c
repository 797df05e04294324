/*
 * CPU oracle for the FP8 (E4M3) 128x128 block-scaled GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file; only the test suite, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header, table or constant with the CUDA
 * library: the E4M3 table below is generated from the bit formula at load time.
 *
 * What it computes, and where that is defined:
 *   - E4M3 format (1 sign / 4 exponent / 3 mantissa bits, largest finite value
 *     about 448): DeepGEMM FP8 write-up (demingchina.com/news/60142) §3.1 format
 *     table; DeepGEMM FP8 library page (2kiu.com/news/5461879) §2.1.
 *   - One FP32 scale per 128x128 block of A and of B, each output block result
 *     multiplied by the matching A-block and B-block scales:
 *     2kiu.com/news/5461879 §2.1 and §3.3 (FP32 scale storage).
 *   - FP8 products accumulated in FP32, long K accumulated in segments
 *     (per-K-block promotion): 2kiu.com/news/5461879 §3.3.
 *   - Scales computed ahead of time from the data range and multiplied back at
 *     the output end: demingchina.com/news/60142 §3.1; dynamic activation
 *     scales: 2kiu.com/news/5461879 §4/§5 (activation scales recomputed per call).
 *
 * Arithmetic is FP64 (see dgo_gemm_ref for why the per-K-block partial is exact).
 * Plain loops; the only parallelism is an OpenMP loop over independent rows.
 *
 * Readings where the pages are silent:
 *   - scale s = fl32(amax / 448) by a correctly rounded division; s = 1 if amax == 0;
 *   - the quantized code is fl32(x / s) rounded to the nearest finite E4M3 value,
 *     ties to the even mantissa code, magnitudes above 448 saturate to 448, the
 *     sign of zero is kept;
 *   - the output is the FP64 block formula rounded once to BF16 (nearest, ties even).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------- */
/* E4M3 decode: byte s|eeee|mmm, exponent bias 7, no infinities, NaN = x1111111 */
/* ------------------------------------------------------------------------- */
double dgo_e4m3_decode(uint8_t b)
{
    int s = (b >> 7) & 1;
    int e = (b >> 3) & 0xF;
    int m = b & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;           /* 0x7F / 0xFF */
    if (e == 0) v = (double)m * ldexp(1.0, -9);     /* subnormal: m/8 * 2^(1-7) */
    else v = (1.0 + (double)m / 8.0) * ldexp(1.0, e - 7);
    return s ? -v : v;
}

void dgo_e4m3_table(double *out256)
{
    for (int b = 0; b < 256; ++b) out256[b] = dgo_e4m3_decode((uint8_t)b);
}

/* Non-negative finite magnitudes, codes 0x00..0x7E, strictly increasing. */
static double g_mag[127];
static int g_mag_ready = 0;

static void init_mag(void)
{
    if (g_mag_ready) return;
    for (int c = 0; c < 127; ++c) g_mag[c] = dgo_e4m3_decode((uint8_t)c);
    g_mag_ready = 1;
}

void dgo_init(void) { init_mag(); }

/* Nearest finite E4M3 code to a float, ties to the even code, saturating. */
uint8_t dgo_e4m3_encode(float v)
{
    init_mag();
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= g_mag[126]) return sign | 126;          /* satfinite: clamp to 448 */
    /* largest code c with g_mag[c] <= a (binary search over 0..125) */
    int lo = 0, hi = 126;                            /* g_mag[lo] <= a < g_mag[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (g_mag[mid] <= a) lo = mid; else hi = mid;
    }
    if (g_mag[lo] == a) return sign | (uint8_t)lo;
    /* the midpoint of two neighbouring E4M3 values is exact in double */
    double midpt = 0.5 * (g_mag[lo] + g_mag[hi]);
    int code;
    if (a < midpt) code = lo;
    else if (a > midpt) code = hi;
    else code = (lo % 2 == 0) ? lo : hi;             /* tie: even mantissa code */
    return sign | (uint8_t)code;
}

void dgo_e4m3_encode_array(const float *v, int64_t n, uint8_t *out)
{
    init_mag();
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = dgo_e4m3_encode(v[i]);
}

/* ------------------------------------------------------------------------- */
/* BF16                                                                       */
/* ------------------------------------------------------------------------- */
static float bf16_bits_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round a double to the nearest BF16 (8 significant bits), ties to even. */
uint16_t dgo_bf16_from_double(double x)
{
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0x0000;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7F80;
    int e;
    frexp(a, &e);                        /* a in [2^(e-1), 2^e) */
    int qexp = (e - 1) - 7;              /* spacing of BF16 values in this binade */
    if (qexp < -133) qexp = -133;        /* subnormal BF16 spacing is 2^-133 */
    double q = ldexp(1.0, qexp);
    double r = a / q;                    /* exact: division by a power of two */
    double fl = floor(r);
    double frac = r - fl;                /* exact */
    if (frac > 0.5 || (frac == 0.5 && fmod(fl, 2.0) != 0.0)) fl += 1.0;
    double res = fl * q;                 /* exact */
    if (res >= ldexp(1.0, 128)) return sign | 0x7F80;
    float f = (float)res;                /* exact: res has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)(u >> 16);
}

void dgo_bf16_from_double_array(const double *x, int64_t n, uint16_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = dgo_bf16_from_double(x[i]);
}

/* ------------------------------------------------------------------------- */
/* Block quantizer: BF16 [R][C] -> E4M3 codes [R][C] + FP32 scales [Rb][Cb]   */
/* ------------------------------------------------------------------------- */
/*
 * Blocks of brows x blk elements: brows = blk is the 128x128 form; brows = 1 gives
 * one scale per row and 128-column group ("per-group, 128 elements a group",
 * demingchina.com/news/60142 §5.2), S [R][Cb].
 */
static void quantize_blocks(const uint16_t *X, int64_t R, int64_t C, int64_t brows, int64_t blk,
                            uint8_t *Q, float *S);

void dgo_quantize_blockwise(const uint16_t *X, int64_t R, int64_t C, int64_t blk,
                            uint8_t *Q, float *S)
{
    quantize_blocks(X, R, C, blk, blk, Q, S);
}

void dgo_quantize_groups(const uint16_t *X, int64_t R, int64_t C, int64_t blk, uint8_t *Q, float *S)
{
    quantize_blocks(X, R, C, 1, blk, Q, S);
}

static void quantize_blocks(const uint16_t *X, int64_t R, int64_t C, int64_t brows, int64_t blk,
                            uint8_t *Q, float *S)
{
    init_mag();
    int64_t Rb = (R + brows - 1) / brows, Cb = (C + blk - 1) / blk;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t br = 0; br < Rb; ++br) {
        int64_t r0 = br * brows, r1 = r0 + brows < R ? r0 + brows : R;
        for (int64_t bc = 0; bc < Cb; ++bc) {
            int64_t c0 = bc * blk, c1 = c0 + blk < C ? c0 + blk : C;
            float amax = 0.0f;
            for (int64_t r = r0; r < r1; ++r)
                for (int64_t c = c0; c < c1; ++c) {
                    float a = fabsf(bf16_bits_to_float(X[r * C + c]));
                    if (a > amax) amax = a;
                }
            /* correctly rounded FP32 division: FP64 quotient of two floats,
               rounded once more to FP32, is the correctly rounded FP32 quotient */
            float s = (amax == 0.0f) ? 1.0f : (float)((double)amax / 448.0);
            S[br * Cb + bc] = s;
            for (int64_t r = r0; r < r1; ++r)
                for (int64_t c = c0; c < c1; ++c) {
                    float x = bf16_bits_to_float(X[r * C + c]);
                    float v = (float)((double)x / (double)s);
                    Q[r * C + c] = dgo_e4m3_encode(v);
                }
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Block-scaled GEMM, C = A * B^T                                             */
/* ------------------------------------------------------------------------- */
/*
 * ref[m][n] = sum over kb (ascending) of
 *             (double)sA[m/128][kb] * (double)sB[n/128][kb] * P_kb[m][n],
 * P_kb[m][n] = sum_{k in kb} dec(A[m][k]) * dec(B[n][k]).
 *
 * P_kb is exact in FP64 in any summation order: every E4M3 value is an integer
 * multiple of 2^-9 with magnitude <= 448, so each product is a multiple of 2^-18
 * below 2^18, and a sum of 128 of them is below 2^25 in magnitude: at most 43
 * significant bits.  The product of two FP32 scales is exact in FP64 (48 bits).
 *
 * A: [M][K] codes, B: [N][K] codes, sA: [ceil(M/128)][ceil(K/128)],
 * sB: [ceil(N/128)][ceil(K/128)].
 * Only rows m in rows[0..nrows) and columns n in cols[0..ncols) are evaluated
 * (pass rows == NULL / cols == NULL for all); out is [nrows][ncols].
 * K need not be a multiple of blk: the last K block then holds the K % blk
 * columns that exist and nothing else (each K step clipped to what remains,
 * demingchina.com/news/60142 §6.3), with its own pair of scales.
 */
static void decode_rows(const uint8_t *X, int64_t K, int64_t row, double *out, const double *tab)
{
    for (int64_t k = 0; k < K; ++k) out[k] = tab[X[row * K + k]];
}

/*
 * The same formula with A's scales per `ablk` rows: sA[m / ablk][kb].  ablk = blk
 * is the 128x128 form above; ablk = 1 gives one scale per row and 128-wide K group
 * ("per-group, 128 elements a group", demingchina.com/news/60142 §5.2), sA [M][Kb].
 */
static void gemm_ref_impl(const uint8_t *A, const float *sA, int64_t ablk, const uint8_t *B, const float *sB,
                          int64_t M, int64_t N, int64_t K, int64_t blk,
                          const int64_t *rows, int64_t nrows, const int64_t *cols, int64_t ncols,
                          double *out);

void dgo_gemm_ref(const uint8_t *A, const float *sA, const uint8_t *B, const float *sB,
                  int64_t M, int64_t N, int64_t K, int64_t blk,
                  const int64_t *rows, int64_t nrows, const int64_t *cols, int64_t ncols,
                  double *out)
{
    gemm_ref_impl(A, sA, blk, B, sB, M, N, K, blk, rows, nrows, cols, ncols, out);
}

void dgo_gemm_ref_rowscale(const uint8_t *A, const float *sA, const uint8_t *B, const float *sB,
                           int64_t M, int64_t N, int64_t K, int64_t blk,
                           const int64_t *rows, int64_t nrows, const int64_t *cols, int64_t ncols,
                           double *out)
{
    gemm_ref_impl(A, sA, 1, B, sB, M, N, K, blk, rows, nrows, cols, ncols, out);
}

static void gemm_ref_impl(const uint8_t *A, const float *sA, int64_t ablk, const uint8_t *B, const float *sB,
                          int64_t M, int64_t N, int64_t K, int64_t blk,
                          const int64_t *rows, int64_t nrows, const int64_t *cols, int64_t ncols,
                          double *out)
{
    double tab[256];
    dgo_e4m3_table(tab);
    int64_t Kb = (K + blk - 1) / blk;
    if (rows == NULL) nrows = M;
    if (cols == NULL) ncols = N;
    /* decode the needed B rows once */
    double *Bd = (double *)malloc((size_t)ncols * (size_t)K * sizeof(double));
    for (int64_t j = 0; j < ncols; ++j) {
        int64_t n = cols ? cols[j] : j;
        decode_rows(B, K, n, Bd + j * K, tab);
    }
#pragma omp parallel
    {
        double *Ad = (double *)malloc((size_t)K * sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < nrows; ++i) {
            int64_t m = rows ? rows[i] : i;
            decode_rows(A, K, m, Ad, tab);
            for (int64_t j = 0; j < ncols; ++j) {
                int64_t n = cols ? cols[j] : j;
                const double *b = Bd + j * K;
                double ref = 0.0;
                for (int64_t kb = 0; kb < Kb; ++kb) {
                    double p = 0.0;
                    int64_t k1 = (kb + 1) * blk < K ? (kb + 1) * blk : K;
                    for (int64_t k = kb * blk; k < k1; ++k) p += Ad[k] * b[k];
                    double s = (double)sA[(m / ablk) * Kb + kb] * (double)sB[(n / blk) * Kb + kb];
                    ref += s * p;
                }
                out[i * ncols + j] = ref;
            }
        }
        free(Ad);
    }
    free(Bd);
}

/*
 * Grouped-contiguous form: the rows of A (and of C) are the concatenation of the
 * experts' token rows, expert g owning rows [off[g], off[g+1]); expert g's weights
 * are B[g] ([N][K] codes) with scales sB[g] ([ceil(N/128)][ceil(K/128)]).  A row that
 * belongs to no expert (beyond off[G]) is left untouched in out.
 * Row m uses the plain dense formula against B[g], sB[g] for the g that owns it.
 * rows[0..nrows) lists the rows to evaluate; cols == NULL means all N columns.
 */
void dgo_grouped_gemm_ref(const uint8_t *A, const float *sA, const uint8_t *B, const float *sB,
                          const int32_t *off, int64_t G, int64_t N, int64_t K, int64_t blk,
                          const int64_t *rows, int64_t nrows, const int64_t *cols, int64_t ncols,
                          double *out)
{
    int64_t Nb = (N + blk - 1) / blk, Kb = (K + blk - 1) / blk;
    if (cols == NULL) ncols = N;
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t m = rows[i];
        int64_t g = -1;
        for (int64_t e = 0; e < G; ++e)
            if (off[e] <= m && m < off[e + 1]) { g = e; break; }
        if (g < 0) continue;
        /* the row's m-block scale row is sA[m/128]; evaluate one row against expert g */
        const uint8_t *Bg = B + g * N * K;
        const float *sBg = sB + g * Nb * Kb;
        int64_t one_row = m;
        /* dgo_gemm_ref indexes A by m and sA by m/blk, so it takes the full A, sA */
        dgo_gemm_ref(A, sA, Bg, sBg, m + 1, N, K, blk, &one_row, 1, cols, ncols, out + i * ncols);
    }
}
