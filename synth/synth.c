/*
 * synth.c -- seeded synthetic inputs for the FP8 block-scaled GEMM.
 *
 * This module only makes inputs.  It holds none of the GEMM's arithmetic:
 * no decode, no product, no accumulation, no output rounding.  Both the CPU
 * oracle's tests and the CUDA path's tests and benchmark draw their inputs
 * from here, so the two sides see the same bytes.
 *
 * Random numbers: a counter-based generator.  Element i of stream s is
 *   splitmix64 finaliser applied to  key(s) + (i + 1) * 0x9E3779B97F4A7C15,
 * key(s) = splitmix64 finaliser of s.  Normals come in pairs from the
 * Box-Muller transform in double precision, rounded once to fp32.
 *
 * Quantisation (the input preparation that the pages leave to the user, see
 * the turtlesai.it summary: casting to FP8 is delegated to developers):
 * per block, amax = max |x| in fp32, scale = amax / 448 (fp32 division),
 * q = e4m3(x / scale) with round-to-nearest-even and saturation at +-448;
 * an all-zero block gets scale 1.  A uses 1x128 blocks with the scales stored
 * column-major (sf[kb * ld + row]); B uses 128x128 blocks, sf[nb][kb].
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SY_BLOCK 128
#define SY_GOLDEN 0x9E3779B97F4A7C15ull

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t stream) { return mix64(stream + SY_GOLDEN); }

uint64_t synth_u64(uint64_t stream, uint64_t index) {
    return mix64(stream_key(stream) + (index + 1) * SY_GOLDEN);
}

/* uniform double in [0, 1) with 53 random bits */
static inline double u01(uint64_t r) { return (double)(r >> 11) * 0x1.0p-53; }

/* standard normal number i of a stream: pair p = i / 2 uses counters 2p, 2p+1 */
static inline float normal_at(uint64_t key, uint64_t i) {
    uint64_t p = i >> 1;
    uint64_t r1 = mix64(key + (2 * p + 1) * SY_GOLDEN);
    uint64_t r2 = mix64(key + (2 * p + 2) * SY_GOLDEN);
    double u1 = 1.0 - u01(r1);          /* (0, 1] so log is finite */
    double u2 = u01(r2);
    double rad = sqrt(-2.0 * log(u1));
    double ang = 6.283185307179586476925286766559 * u2;
    double z = (i & 1) ? rad * sin(ang) : rad * cos(ang);
    return (float)z;
}

void synth_normal_f32(uint64_t stream, uint64_t offset, long n, float *out) {
    uint64_t key = stream_key(stream);
    #pragma omp parallel for schedule(static)
    for (long i = 0; i < n; ++i) out[i] = normal_at(key, offset + (uint64_t)i);
}

void synth_uniform_f64(uint64_t stream, uint64_t offset, long n, double *out) {
    for (long i = 0; i < n; ++i) out[i] = u01(synth_u64(stream, offset + (uint64_t)i));
}

/* e4m3 ("fn") encoder with round-to-nearest-even and saturation to +-448.
 * Written from the format: 3 mantissa bits, exponent bias 7, subnormal quantum
 * 2^-9, largest finite 448 = 1.75 * 2^8.  NaN input maps to the NaN code 0x7F
 * (never produced by the generator). */
uint8_t synth_e4m3_encode(float xf) {
    double x = (double)xf;
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= 448.0) return sign | 0x7E;          /* saturate (also +-inf) */
    if (a == 0.0) return sign;
    int e;
    (void)frexp(a, &e);                 /* a in [2^(e-1), 2^e) */
    int q = e - 4;                      /* quantum for 4 significant bits */
    if (q < -9) q = -9;                 /* subnormal quantum */
    double r = nearbyint(ldexp(a, -q)); /* ties to even */
    double y = ldexp(r, q);
    if (y > 448.0) y = 448.0;           /* cannot happen below 448, kept for clarity */
    if (y == 0.0) return sign;
    /* pack y: exact e4m3 value */
    int ey;
    double fy = frexp(y, &ey);          /* y = fy * 2^ey, fy in [0.5, 1) */
    int biased = ey - 1 + 7;            /* y = 1.f * 2^(ey-1) */
    uint8_t code;
    if (biased <= 0) {                  /* subnormal: y = m/8 * 2^-6 */
        int m = (int)ldexp(y, 9);
        code = (uint8_t)m;
    } else {
        int m = (int)((fy * 2.0 - 1.0) * 8.0);
        code = (uint8_t)((biased << 3) | m);
    }
    return sign | code;
}

/* e5m2 encoder with round-to-nearest-even and saturation to +-57344.
 * Written from the format: 2 mantissa bits, exponent bias 15, subnormal quantum
 * 2^-16, largest finite 57344 = 1.75 * 2^15 (code 0x7B; 0x7C is infinity).
 * NaN input maps to a NaN code (never produced by the generator). */
uint8_t synth_e5m2_encode(float xf) {
    double x = (double)xf;
    if (isnan(x)) return 0x7E;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= 57344.0) return sign | 0x7B;        /* saturate (also +-inf) */
    if (a == 0.0) return sign;
    int e;
    (void)frexp(a, &e);                 /* a in [2^(e-1), 2^e) */
    int q = e - 3;                      /* quantum for 3 significant bits */
    if (q < -16) q = -16;               /* subnormal quantum */
    double r = nearbyint(ldexp(a, -q)); /* ties to even */
    double y = ldexp(r, q);
    if (y > 57344.0) y = 57344.0;
    if (y == 0.0) return sign;
    int ey;
    double fy = frexp(y, &ey);          /* y = fy * 2^ey, fy in [0.5, 1) */
    int biased = ey - 1 + 15;
    uint8_t code;
    if (biased <= 0) {                  /* subnormal: y = m/4 * 2^-14 = m * 2^-16 */
        code = (uint8_t)(int)ldexp(y, 16);
    } else {
        int m = (int)((fy * 2.0 - 1.0) * 4.0);
        code = (uint8_t)((biased << 2) | m);
    }
    return sign | code;
}

/* fmt 0: e4m3 (largest finite 448), 1: e5m2 (largest finite 57344) */
static inline uint8_t encode_fmt(float v, int fmt) {
    return fmt == 0 ? synth_e4m3_encode(v) : synth_e5m2_encode(v);
}

static inline float block_scale_fmt(float amax, int fmt) {
    const float top = fmt == 0 ? 448.0f : 57344.0f;
    return amax > 0.0f ? amax / top : 1.0f;
}

static inline float block_scale(float amax) {
    return block_scale_fmt(amax, 0);
}

/* Quantise rows x[rows][K] (fp32) with 1x128 blocks.
 * q[rows][K] codes; sf[kb * ld + r] scales (column-major, ld >= rows). */
void synth_quantize_1x128(const float *x, long rows, int K, uint8_t *q, float *sf, long ld) {
    const int KB = (K + SY_BLOCK - 1) / SY_BLOCK;
    #pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        const float *xr = x + r * (long)K;
        uint8_t *qr = q + r * (long)K;
        for (int kb = 0; kb < KB; ++kb) {
            int k0 = kb * SY_BLOCK, k1 = k0 + SY_BLOCK < K ? k0 + SY_BLOCK : K;
            float amax = 0.0f;
            for (int k = k0; k < k1; ++k) { float v = fabsf(xr[k]); if (v > amax) amax = v; }
            float s = block_scale(amax);
            for (int k = k0; k < k1; ++k) qr[k] = synth_e4m3_encode(xr[k] / s);
            sf[(long)kb * ld + r] = s;
        }
    }
}

/* Quantise x[rows][K] with 128x128 blocks; sf[nb][kb] row-major. */
void synth_quantize_128x128(const float *x, long rows, int K, uint8_t *q, float *sf) {
    const int KB = (K + SY_BLOCK - 1) / SY_BLOCK;
    const long RB = (rows + SY_BLOCK - 1) / SY_BLOCK;
    #pragma omp parallel for collapse(2) schedule(static)
    for (long rb = 0; rb < RB; ++rb) {
        for (int kb = 0; kb < KB; ++kb) {
            long r0 = rb * SY_BLOCK, r1 = r0 + SY_BLOCK < rows ? r0 + SY_BLOCK : rows;
            int k0 = kb * SY_BLOCK, k1 = k0 + SY_BLOCK < K ? k0 + SY_BLOCK : K;
            float amax = 0.0f;
            for (long r = r0; r < r1; ++r)
                for (int k = k0; k < k1; ++k) { float v = fabsf(x[r * K + k]); if (v > amax) amax = v; }
            float s = block_scale(amax);
            for (long r = r0; r < r1; ++r)
                for (int k = k0; k < k1; ++k) q[r * K + k] = synth_e4m3_encode(x[r * K + k] / s);
            sf[rb * KB + kb] = s;
        }
    }
}

/* Fused generate + quantise, so that large operands need no fp32 copy.
 * Element (r, k) of the matrix is normal number offset + r*K + k of `stream`,
 * optionally multiplied (in fp32) by row_scale[r] before quantisation.
 * mode 0: 1x128 blocks, column-major scales sf[kb*ld + r] (A operand);
 * mode 1: 128x128 blocks, sf[rb][kb] (B operand). */
void synth_quantized_matrix(uint64_t stream, uint64_t offset, long rows, int K,
                            const float *row_scale, int mode,
                            uint8_t *q, float *sf, long ld, int fmt) {
    const int KB = (K + SY_BLOCK - 1) / SY_BLOCK;
    uint64_t key = stream_key(stream);
    if (mode == 0) {
        #pragma omp parallel
        {
            float buf[SY_BLOCK];
            #pragma omp for schedule(static)
            for (long r = 0; r < rows; ++r) {
                float rs = row_scale ? row_scale[r] : 1.0f;
                for (int kb = 0; kb < KB; ++kb) {
                    int k0 = kb * SY_BLOCK, k1 = k0 + SY_BLOCK < K ? k0 + SY_BLOCK : K;
                    float amax = 0.0f;
                    for (int k = k0; k < k1; ++k) {
                        float v = normal_at(key, offset + (uint64_t)(r * K + k));
                        if (row_scale) v = v * rs;
                        buf[k - k0] = v;
                        float a = fabsf(v); if (a > amax) amax = a;
                    }
                    float s = block_scale_fmt(amax, fmt);
                    for (int k = k0; k < k1; ++k) q[r * K + k] = encode_fmt(buf[k - k0] / s, fmt);
                    sf[(long)kb * ld + r] = s;
                }
            }
        }
    } else {
        const long RB = (rows + SY_BLOCK - 1) / SY_BLOCK;
        #pragma omp parallel
        {
            static __thread float tile[SY_BLOCK * SY_BLOCK];
            #pragma omp for collapse(2) schedule(static)
            for (long rb = 0; rb < RB; ++rb) {
                for (int kb = 0; kb < KB; ++kb) {
                    long r0 = rb * SY_BLOCK, r1 = r0 + SY_BLOCK < rows ? r0 + SY_BLOCK : rows;
                    int k0 = kb * SY_BLOCK, k1 = k0 + SY_BLOCK < K ? k0 + SY_BLOCK : K;
                    float amax = 0.0f;
                    for (long r = r0; r < r1; ++r) {
                        float rs = row_scale ? row_scale[r] : 1.0f;
                        for (int k = k0; k < k1; ++k) {
                            float v = normal_at(key, offset + (uint64_t)(r * K + k));
                            if (row_scale) v = v * rs;
                            tile[(r - r0) * SY_BLOCK + (k - k0)] = v;
                            float a = fabsf(v); if (a > amax) amax = a;
                        }
                    }
                    float s = block_scale_fmt(amax, fmt);
                    for (long r = r0; r < r1; ++r)
                        for (int k = k0; k < k1; ++k)
                            q[r * K + k] = encode_fmt(tile[(r - r0) * SY_BLOCK + (k - k0)] / s, fmt);
                    sf[rb * KB + kb] = s;
                }
            }
        }
    }
}
