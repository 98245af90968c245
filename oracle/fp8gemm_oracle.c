/*
 * fp8gemm_oracle.c -- CPU oracle for the FP8 (e4m3) block-scaled NT GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, obviously-correct
 * definition that the CUDA library is checked against.  Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg load it.  It shares no code,
 * header, table or constant with the CUDA library under moe_grouped_gemm_08_b200/.
 *
 * What it computes (sources, by page and section):
 *   - "DeepGEMM" product page (flashmla.org), section "What is DeepGEMM":
 *     an FP8 GEMM library with one normal (dense) layout and two MoE layouts,
 *     contiguous and masked.
 *   - "DeepGEMM" how-to (aisharenet.com), section "Main functions" 1-3:
 *     gemm_fp8_fp8_bf16_nt, m_grouped_gemm_fp8_fp8_bf16_nt_contiguous and
 *     m_grouped_gemm_fp8_fp8_bf16_nt_masked; FP8 inputs, BF16 output.
 *   - "DeepGEMM: Efficienza e Precisione..." (turtlesai.it), summary paragraph:
 *     NT layout only (LHS not transposed, RHS transposed), fine-grained
 *     scaling, two-level accumulation on CUDA cores.
 *   - DeepSeek DeepGEMM news article (senqingzn.com), optimisation paragraph:
 *     the FP8 tensor-core accumulation is not precise enough, so partial sums
 *     are promoted into a higher-precision accumulator.
 * Operands are e4m3 codes by default; either operand may instead be e5m2
 * (the how-to, "Main functions": E4M3 or E5M2 inputs).
 * The pages leave the scale granularities open.  This oracle takes 1x128
 * (one fp32 scale per row of A per 128-wide K block, stored column-major with
 * leading dimension ld) and 128x128 (one fp32 scale per 128x128 block of B).
 *
 * Definition, for every output element:
 *   S_kb   = sum_{k in block kb} dec(A[m,k]) * dec(B[n,k])        (fp64, exact)
 *   C[m,n] = bf16_rne( sum_kb S_kb * (sfa[kb][m] * sfb[n/128][kb]) )  (fp64)
 * Every e4m3 product is a multiple of 2^-18 below 2^18 in magnitude, so a sum
 * of at most 128 of them needs fewer than 44 significant bits and S_kb is exact
 * in fp64.  The product of two fp32 scales is exact in fp64 (48 bits).  The
 * only roundings are the fp64 scale multiply, the fp64 accumulation over kb
 * (in ascending kb order) and the single final rounding to bf16.
 *
 * It also defines the cast step that produces those inputs from BF16 values
 * (oracle_quantize_rows / oracle_quantize_blocks, see below).
 *
 * Build: plain C11, -ffp-contract=off, OpenMP over output rows.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORC_BLOCK 128

/* ---------------------------------------------------------------------------
 * e4m3 ("fn" variant) decode table, built from the format definition:
 * 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0
 * encodes subnormals m/8 * 2^-6; S.1111.111 is NaN; there is no infinity, so
 * the largest finite magnitude is 1.75 * 2^8 = 448.
 * ------------------------------------------------------------------------- */
static double g_dec[256];
static int g_dec_ready = 0;

static void build_decode_table(void) {
    for (int code = 0; code < 256; ++code) {
        int sign = (code >> 7) & 1;
        int e = (code >> 3) & 0xF;
        int m = code & 0x7;
        double v;
        if (e == 0xF && m == 0x7) {
            v = NAN;
        } else if (e == 0) {
            v = ldexp((double)m / 8.0, -6);
        } else {
            v = ldexp(1.0 + (double)m / 8.0, e - 7);
        }
        g_dec[code] = sign ? -v : v;
    }
    g_dec_ready = 1;
}

static const double *dec_table(void) {
    if (!g_dec_ready) build_decode_table();
    return g_dec;
}

/* ---------------------------------------------------------------------------
 * e5m2 decode table, from the format definition: 1 sign bit, 5 exponent bits
 * with bias 15, 2 mantissa bits; exponent field 0 encodes subnormals
 * m/4 * 2^-14; exponent field 31 encodes infinity (m = 0) and NaN.  The
 * largest finite magnitude is 1.75 * 2^15 = 57344.  ("DeepGEMM" how-to,
 * aisharenet.com, "Main functions": the FP8 inputs are E4M3 or E5M2.)
 * ------------------------------------------------------------------------- */
static double g_dec52[256];
static int g_dec52_ready = 0;

static void build_decode_table_e5m2(void) {
    for (int code = 0; code < 256; ++code) {
        int sign = (code >> 7) & 1;
        int e = (code >> 2) & 0x1F;
        int m = code & 0x3;
        double v;
        if (e == 0x1F) {
            v = m == 0 ? INFINITY : NAN;
        } else if (e == 0) {
            v = ldexp((double)m / 4.0, -14);
        } else {
            v = ldexp(1.0 + (double)m / 4.0, e - 15);
        }
        g_dec52[code] = sign ? -v : v;
    }
    g_dec52_ready = 1;
}

/* fmt 0: e4m3, 1: e5m2 */
static const double *dec_table_fmt(int fmt) {
    if (fmt == 0) return dec_table();
    if (!g_dec52_ready) build_decode_table_e5m2();
    return g_dec52;
}

/* Build both decode tables before a parallel region (they are filled lazily, once). */
static void tables_ready(void) {
    (void)dec_table();
    (void)dec_table_fmt(1);
}

void oracle_e5m2_decode_table(double *out256) {
    memcpy(out256, dec_table_fmt(1), 256 * sizeof(double));
}

/* Every finite code of a format is an integer multiple of the format's quantum:
 * 2^-9 for e4m3, 2^-16 for e5m2.  Products of e5m2 codes span more than 53 bits,
 * so K-block sums that involve e5m2 are formed exactly in 128-bit integers in
 * these units and converted to fp64 once (one rounding, relative 2^-53). */
static int quantum_exp(int fmt) { return fmt == 0 ? 9 : 16; }

static int64_t code_units(int fmt, uint8_t code) {
    double v = dec_table_fmt(fmt)[code];
    if (!isfinite(v)) return 0;  /* non-finite codes take the fp64 path in row_nt */
    return (int64_t)ldexp(v, quantum_exp(fmt));
}

void oracle_e4m3_decode_table(double *out256) {
    memcpy(out256, dec_table(), sizeof(double) * 256);
}

/* ---------------------------------------------------------------------------
 * fp64 -> bf16 with one round-to-nearest-even step.
 * bf16 = 1 sign, 8 exponent (bias 127), 7 mantissa bits: 8 significant bits
 * for normals, a fixed quantum of 2^-133 below 2^-126, overflow to infinity.
 * Output: the bf16 bit pattern.
 * ------------------------------------------------------------------------- */
uint16_t oracle_bf16_from_f64(double x) {
    if (isnan(x)) return (uint16_t)(signbit(x) ? 0xFFC0u : 0x7FC0u);
    if (isinf(x)) return (uint16_t)(signbit(x) ? 0xFF80u : 0x7F80u);
    if (x == 0.0) return (uint16_t)(signbit(x) ? 0x8000u : 0x0000u);
    int e;
    (void)frexp(x, &e);            /* |x| in [2^(e-1), 2^e) */
    int q = e - 8;                 /* quantum of an 8-significant-bit number */
    if (q < -133) q = -133;        /* bf16 subnormal quantum */
    double scaled = ldexp(x, -q);  /* exact: power-of-two rescale */
    double r = nearbyint(scaled);  /* default rounding mode: to nearest, ties even */
    double y = ldexp(r, q);
    if (fabs(y) >= ldexp(1.0, 128)) return (uint16_t)(signbit(x) ? 0xFF80u : 0x7F80u);
    float yf = (float)y;           /* exact: y has at most 8 significant bits */
    uint32_t bits;
    memcpy(&bits, &yf, sizeof bits);
    return (uint16_t)(bits >> 16);
}

/* ---------------------------------------------------------------------------
 * One output row of the dense NT product (the definition above).
 *   a_row : K e4m3 codes of row m of A
 *   sfa_m : sfa + m, stepping by ld between K blocks (column-major scales)
 *   B     : N x K e4m3 codes, row-major
 *   sfb   : ceil(N/128) x ceil(K/128) fp32, row-major
 *   c_row : N bf16 outputs; acc_row (optional) receives the fp64 pre-rounding value
 * ------------------------------------------------------------------------- */
static void row_nt(const uint8_t *a_row, const float *sfa_m, long ld,
                   const uint8_t *B, const float *sfb, int N, int K,
                   uint16_t *c_row, double *acc_row, int fa, int fb) {
    const double *dec = dec_table();
    const double *deca = dec_table_fmt(fa), *decb = dec_table_fmt(fb);
    const int KB = (K + ORC_BLOCK - 1) / ORC_BLOCK;
    int64_t ua[256], ub[256];
    if (fa != 0 || fb != 0)
        for (int c = 0; c < 256; ++c) { ua[c] = code_units(fa, (uint8_t)c); ub[c] = code_units(fb, (uint8_t)c); }
    for (int n = 0; n < N; ++n) {
        const uint8_t *b_row = B + (size_t)n * K;
        double acc = 0.0;
        for (int kb = 0; kb < KB; ++kb) {
            int k0 = kb * ORC_BLOCK;
            int k1 = k0 + ORC_BLOCK < K ? k0 + ORC_BLOCK : K;
            double s = 0.0;
            if (fa == 0 && fb == 0) {
                for (int k = k0; k < k1; ++k) s += dec[a_row[k]] * dec[b_row[k]];
            } else {
                /* a block holding a non-finite code (e4m3 NaN; e5m2 infinity or NaN) is summed in
                 * fp64: the IEEE result (NaN, or an infinity) does not depend on the finite terms'
                 * rounding; every other block exactly, in quanta */
                int special = 0;
                for (int k = k0; k < k1 && !special; ++k)
                    special = !isfinite(deca[a_row[k]]) || !isfinite(decb[b_row[k]]);
                if (special) {
                    for (int k = k0; k < k1; ++k) s += deca[a_row[k]] * decb[b_row[k]];
                } else {
                    __int128 t = 0;
                    for (int k = k0; k < k1; ++k) t += (__int128)ua[a_row[k]] * ub[b_row[k]];
                    s = ldexp((double)t, -(quantum_exp(fa) + quantum_exp(fb)));
                }
            }
            double scale = (double)sfa_m[(size_t)kb * ld] *
                           (double)sfb[(size_t)(n / ORC_BLOCK) * KB + kb];
            acc += s * scale;
        }
        c_row[n] = oracle_bf16_from_f64(acc);
        if (acc_row) acc_row[n] = acc;
    }
}

/* Dense: C[M,N] = A[M,K] . B[N,K]^T with sfa[KB][ld] and sfb[NB][KB].
 * acc (optional, M x N fp64) receives the unrounded values. */
void oracle_gemm_nt(const uint8_t *A, const float *sfa, long ld,
                    const uint8_t *B, const float *sfb,
                    int M, int N, int K, uint16_t *C, double *acc, int fa, int fb) {
    tables_ready();
    #pragma omp parallel for schedule(dynamic, 1)
    for (int m = 0; m < M; ++m)
        row_nt(A + (size_t)m * K, sfa + m, ld, B, sfb, N, K,
               C + (size_t)m * N, acc ? acc + (size_t)m * N : NULL, fa, fb);
}

/* Dense, selected rows only: row rows[i] of the product goes to C[i,:].
 * Used to check large products on a sample of rows. */
void oracle_gemm_nt_rows(const uint8_t *A, const float *sfa, long ld,
                         const uint8_t *B, const float *sfb,
                         int M, int N, int K, const int *rows, int nrows,
                         uint16_t *C, double *acc, int fa, int fb) {
    (void)M;
    tables_ready();
    #pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < nrows; ++i) {
        int m = rows[i];
        row_nt(A + (size_t)m * K, sfa + m, ld, B, sfb, N, K,
               C + (size_t)i * N, acc ? acc + (size_t)i * N : NULL, fa, fb);
    }
}

/* M-grouped contiguous layout ("DeepGEMM" how-to, aisharenet.com, "Main
 * functions" 2; news article, senqingzn.com, MoE-layout paragraph): the rows
 * of all experts are concatenated along M; m_indices[m] names the expert of
 * row m, or is -1 for a padding row.  Row m uses B[g] (N x K) and sfb[g].
 * Rows whose index is -1 (or outside [0,G)) are not written.
 * rows/nrows: optional subset (NULL = all M_total rows, C indexed by m).
 * With a subset, row rows[i] goes to C[i,:]. */
void oracle_grouped_contiguous(const uint8_t *A, const float *sfa, long ld,
                               const uint8_t *B, const float *sfb,
                               const int *m_indices, int M_total, int G,
                               int N, int K, const int *rows, int nrows,
                               uint16_t *C, double *acc, int fa, int fb) {
    const int KB = (K + ORC_BLOCK - 1) / ORC_BLOCK;
    const int NB = (N + ORC_BLOCK - 1) / ORC_BLOCK;
    int count = rows ? nrows : M_total;
    tables_ready();
    #pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < count; ++i) {
        int m = rows ? rows[i] : i;
        int g = m_indices[m];
        if (g < 0 || g >= G) continue;
        row_nt(A + (size_t)m * K, sfa + m, ld,
               B + (size_t)g * N * K, sfb + (size_t)g * NB * KB, N, K,
               C + (size_t)i * N, acc ? acc + (size_t)i * N : NULL, fa, fb);
    }
}

/* M-grouped masked layout ("DeepGEMM" how-to, aisharenet.com, "Main functions"
 * 3; news article, senqingzn.com, decode paragraph): A is [G][Mmax][K],
 * sfa is [G][KB][ld], C is [G][Mmax][N]; group g has masked_m[g] valid rows,
 * which use B[g] and sfb[g].  Rows at or past masked_m[g] are not written. */
void oracle_grouped_masked(const uint8_t *A, const float *sfa, long ld,
                           const uint8_t *B, const float *sfb,
                           const int *masked_m, int G, int Mmax, int N, int K,
                           uint16_t *C, double *acc, int fa, int fb) {
    const int KB = (K + ORC_BLOCK - 1) / ORC_BLOCK;
    const int NB = (N + ORC_BLOCK - 1) / ORC_BLOCK;
    long total = (long)G * Mmax;
    tables_ready();
    #pragma omp parallel for schedule(dynamic, 1)
    for (long gm = 0; gm < total; ++gm) {
        int g = (int)(gm / Mmax);
        int m = (int)(gm % Mmax);
        int valid = masked_m[g];
        if (valid > Mmax) valid = Mmax;
        if (m >= valid) continue;
        row_nt(A + ((size_t)g * Mmax + m) * K, sfa + (size_t)g * KB * ld + m, ld,
               B + (size_t)g * N * K, sfb + (size_t)g * NB * KB, N, K,
               C + ((size_t)g * Mmax + m) * N,
               acc ? acc + ((size_t)g * Mmax + m) * N : NULL, fa, fb);
    }
}

/* ---------------------------------------------------------------------------
 * The cast step before the GEMM: BF16 values to e4m3 codes with fine-grained
 * fp32 scales.  The pages leave this step to the user (turtlesai.it summary:
 * the LHS scales must be laid out for aligned TMA loads, with the FP8 casting
 * done separately; news article, senqingzn.com: fine-grained scaling).  The
 * reading taken here, per block (1 x 128 of a row for A, 128 x 128 for B):
 *   amax  = max |x| over the block (fp32; bf16 -> fp32 is exact)
 *   scale = amax / top in fp32 (one IEEE round-to-nearest division), or 1 if
 *           amax == 0, top = 448 for e4m3 and 57344 for e5m2 (the formats'
 *           largest finite values)
 *   code  = round-to-nearest-even of the fp32 quotient x / scale in the target
 *           format, saturating at +-top
 * ------------------------------------------------------------------------- */

/* e4m3 code of the finite fp32 value v: the nearest of the 127 non-negative
 * finite magnitudes of the decode table (increasing with the code), ties to
 * the even code (mantissa LSB 0), magnitudes above 448 clamped to 448. */
uint8_t oracle_e4m3_encode(float v) {
    const double *dec = dec_table();
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    const double a = fabs((double)v);
    if (a >= dec[0x7E]) return sign | 0x7E;
    int lo = 0, hi = 0x7E;                 /* dec[lo] <= a < dec[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (dec[mid] <= a) lo = mid; else hi = mid;
    }
    const double dl = a - dec[lo], dh = dec[hi] - a;
    int c;
    if (dl < dh) c = lo;
    else if (dh < dl) c = hi;
    else c = (lo % 2 == 0) ? lo : hi;      /* tie: even mantissa */
    return sign | (uint8_t)c;
}

void oracle_e4m3_encode_array(const float *v, long n, uint8_t *out) {
    for (long i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(v[i]);
}

/* e5m2 code of the finite fp32 value v: the nearest of the 124 non-negative finite
 * magnitudes of the e5m2 table (codes 0x00..0x7B, increasing with the code), ties
 * to the even code, magnitudes above 57344 clamped to 57344. */
uint8_t oracle_e5m2_encode(float v) {
    const double *dec = dec_table_fmt(1);
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    const double a = fabs((double)v);
    if (a >= dec[0x7B]) return sign | 0x7B;
    int lo = 0, hi = 0x7B;                 /* dec[lo] <= a < dec[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (dec[mid] <= a) lo = mid; else hi = mid;
    }
    const double dl = a - dec[lo], dh = dec[hi] - a;
    int c;
    if (dl < dh) c = lo;
    else if (dh < dl) c = hi;
    else c = (lo & 1) ? hi : lo;           /* tie: the even code */
    return sign | (uint8_t)c;
}

void oracle_e5m2_encode_array(const float *v, long n, uint8_t *out) {
    for (long i = 0; i < n; ++i) out[i] = oracle_e5m2_encode(v[i]);
}

/* the cast's target format: fmt 0 e4m3 (largest finite 448), 1 e5m2 (57344) */
static uint8_t encode_fmt(float v, int fmt) { return fmt == 0 ? oracle_e4m3_encode(v) : oracle_e5m2_encode(v); }

static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static float block_scale(float amax, int fmt) {
    volatile float s = fmt == 0 ? amax / 448.0f : amax / 57344.0f;  /* one fp32 division */
    return amax == 0.0f ? 1.0f : s;
}

/* A side: X is [G][M][K] bf16 (bit patterns), Q the e4m3 codes in the same
 * layout, sfa the scales [G][ceil(K/128)][ld], ld >= M (rows M..ld-1 of each
 * column are not written). */
void oracle_quantize_rows(const uint16_t *X, int G, int M, int K, uint8_t *Q, float *sfa, long ld, int fmt) {
    const int KB = (K + ORC_BLOCK - 1) / ORC_BLOCK;
    long rows = (long)G * M;
    tables_ready();
    #pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        const int g = (int)(r / M), m = (int)(r % M);
        const uint16_t *x = X + (size_t)r * K;
        uint8_t *q = Q + (size_t)r * K;
        for (int kb = 0; kb < KB; ++kb) {
            const int k0 = kb * ORC_BLOCK, k1 = (k0 + ORC_BLOCK < K) ? k0 + ORC_BLOCK : K;
            float amax = 0.0f;
            for (int k = k0; k < k1; ++k) {
                float a = fabsf(bf16_to_f32(x[k]));
                if (a > amax) amax = a;
            }
            const float s = block_scale(amax, fmt);
            sfa[((size_t)g * KB + kb) * ld + m] = s;
            for (int k = k0; k < k1; ++k) {
                volatile float v = bf16_to_f32(x[k]) / s;   /* one fp32 division */
                q[k] = encode_fmt(v, fmt);
            }
        }
    }
}

/* B side: X is [G][N][K] bf16, Q the codes, sfb the scales [G][ceil(N/128)][ceil(K/128)]. */
void oracle_quantize_blocks(const uint16_t *X, int G, int N, int K, uint8_t *Q, float *sfb, int fmt) {
    const int KB = (K + ORC_BLOCK - 1) / ORC_BLOCK;
    const int NB = (N + ORC_BLOCK - 1) / ORC_BLOCK;
    long blocks = (long)G * NB * KB;
    tables_ready();
    #pragma omp parallel for schedule(static)
    for (long b = 0; b < blocks; ++b) {
        const int g = (int)(b / ((long)NB * KB));
        const int nb = (int)((b / KB) % NB), kb = (int)(b % KB);
        const int n0 = nb * ORC_BLOCK, n1 = (n0 + ORC_BLOCK < N) ? n0 + ORC_BLOCK : N;
        const int k0 = kb * ORC_BLOCK, k1 = (k0 + ORC_BLOCK < K) ? k0 + ORC_BLOCK : K;
        const uint16_t *x = X + (size_t)g * N * K;
        uint8_t *q = Q + (size_t)g * N * K;
        float amax = 0.0f;
        for (int n = n0; n < n1; ++n)
            for (int k = k0; k < k1; ++k) {
                float a = fabsf(bf16_to_f32(x[(size_t)n * K + k]));
                if (a > amax) amax = a;
            }
        const float s = block_scale(amax, fmt);
        sfb[b] = s;
        for (int n = n0; n < n1; ++n)
            for (int k = k0; k < k1; ++k) {
                volatile float v = bf16_to_f32(x[(size_t)n * K + k]) / s;
                q[(size_t)n * K + k] = encode_fmt(v, fmt);
            }
    }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
