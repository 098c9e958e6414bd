/* Host-side seeded generator for the synthetic expert weights.
 *
 * Counter-based, so that any single expert (or any single element) can be
 * regenerated on its own, on the host here and on the GPU by philox_gpu.cu,
 * with identical bits.  Both files implement the same published definitions:
 *
 *   Philox4x32-10: J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw,
 *   "Parallel random numbers: as easy as 1, 2, 3", SC'11, section 3.1
 *   (multipliers 0xD2511F53 / 0xCD9E8D57, Weyl key increments 0x9E3779B9 /
 *   0xBB67AE85, ten rounds).
 *
 *   Bell-shaped values: the sum of the eight 16-bit halves of one Philox
 *   output block (an Irwin-Hall sum of 8 discrete uniforms), centred and
 *   scaled to unit variance in fp64.  Mean 0, sd 1, support +-4.9 sd.  All
 *   steps are exact integer work or single IEEE roundings, so the value is
 *   reproducible bit for bit on any IEEE machine.
 *
 * Element i of stream (k0, k1) uses counter (lo32(i), hi32(i), 0, 0).
 *
 * This is input generation only: it holds none of the MoE layer's arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static inline uint32_t mulhilo32(uint32_t a, uint32_t b, uint32_t *hi) {
    uint64_t p = (uint64_t)a * (uint64_t)b;
    *hi = (uint32_t)(p >> 32);
    return (uint32_t)p;
}

static inline void philox_10(uint32_t c[4], uint32_t k0, uint32_t k1) {
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        uint32_t hi0, hi1;
        uint32_t lo0 = mulhilo32(0xD2511F53u, c[0], &hi0);
        uint32_t lo1 = mulhilo32(0xCD9E8D57u, c[2], &hi1);
        uint32_t n0 = hi1 ^ c[1] ^ k0;
        uint32_t n2 = hi0 ^ c[3] ^ k1;
        c[0] = n0;
        c[1] = lo1;
        c[2] = n2;
        c[3] = lo0;
    }
}

/* Raw block function, exported for known-answer tests. */
void moegen_philox4x32_10(const uint32_t in[4], uint32_t k0, uint32_t k1, uint32_t out[4]) {
    uint32_t c[4] = {in[0], in[1], in[2], in[3]};
    philox_10(c, k0, k1);
    memcpy(out, c, sizeof c);
}

/* Unit-variance value for element i (see header). */
static inline double unit_value(uint64_t i, uint32_t k0, uint32_t k1, double c8) {
    uint32_t c[4] = {(uint32_t)i, (uint32_t)(i >> 32), 0u, 0u};
    philox_10(c, k0, k1);
    int64_t s = 0;
    for (int j = 0; j < 4; ++j) s += (int64_t)(c[j] & 0xFFFFu) + (int64_t)(c[j] >> 16);
    /* 8 * 65535 / 2 = 262140 is the mean; the variance is 8*(65536^2-1)/12. */
    return (double)(s - 262140) * c8;
}

static double unit_scale(void) { return 1.0 / sqrt(2863311530.0); }

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t b;
    memcpy(&b, &f, 4);
    if ((b & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((b >> 16) | 0x40u);
    b += 0x7FFFu + ((b >> 16) & 1u);
    return (uint16_t)(b >> 16);
}

/* float -> OCP e4m3 (fn variant: no infinities, max 448), round to nearest
 * even, saturating to +-448. */
static uint8_t f32_to_e4m3_rne(float f) {
    uint8_t sign = signbit(f) ? 0x80 : 0x00;
    float a = fabsf(f);
    if (!(a == a)) return 0x7F;
    if (a >= 448.0f) return sign | 0x7E;
    if (a < 0.015625f) {                   /* below 2^-6: subnormal, step 2^-9 */
        float m = nearbyintf(a * 512.0f);  /* exact scaling, RNE to integer */
        return sign | (uint8_t)m;          /* m == 8 encodes 2^-6 correctly */
    }
    int e;
    frexpf(a, &e);                         /* a in [2^(e-1), 2^e) */
    int E = e - 1;                         /* unbiased exponent, -6..8 */
    float q = nearbyintf(ldexpf(a, 3 - E)); /* 1.mmm scaled to [8, 16] */
    if (q == 16.0f) {
        q = 8.0f;
        E += 1;
    }
    if (E > 8 || (E == 8 && q > 14.0f)) return sign | 0x7E;
    return sign | (uint8_t)(((E + 7) << 3) | ((int)q - 8));
}

void moegen_f32_to_e4m3(const float *in, uint8_t *out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_e4m3_rne(in[i]);
}

void moegen_f32_to_bf16(const float *in, uint16_t *out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(in[i]);
}

void moegen_normal_f32(float *out, int64_t n, uint32_t k0, uint32_t k1, double sigma) {
    const double c8 = unit_scale();
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (float)(unit_value((uint64_t)i, k0, k1, c8) * sigma);
}

void moegen_normal_bf16(uint16_t *out, int64_t n, uint32_t k0, uint32_t k1, double sigma) {
    const double c8 = unit_scale();
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = f32_to_bf16_rne((float)(unit_value((uint64_t)i, k0, k1, c8) * sigma));
}

/* Row-major [rows, cols] fp32 values, quantised per 128x128 block:
 * s = amax / 448 (fp32; 1 for an all-zero block), q = e4m3(clamp(v / s)).
 * scales is [ceil(rows/128), ceil(cols/128)] row-major.  The weight the
 * tensor stands for is q * s. */
void moegen_e4m3_blocks(uint8_t *q, float *scales, int64_t rows, int64_t cols,
                        uint32_t k0, uint32_t k1, double sigma) {
    const double c8 = unit_scale();
    const int64_t rb = (rows + 127) / 128, cb = (cols + 127) / 128;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b = 0; b < rb * cb; ++b) {
        const int64_t r0 = (b / cb) * 128, c0 = (b % cb) * 128;
        const int64_t r1 = r0 + 128 < rows ? r0 + 128 : rows;
        const int64_t c1 = c0 + 128 < cols ? c0 + 128 : cols;
        float amax = 0.0f;
        for (int64_t r = r0; r < r1; ++r)
            for (int64_t c = c0; c < c1; ++c) {
                float v = (float)(unit_value((uint64_t)(r * cols + c), k0, k1, c8) * sigma);
                float a = fabsf(v);
                if (a > amax) amax = a;
            }
        float s = amax / 448.0f;
        if (amax == 0.0f) s = 1.0f;
        scales[b] = s;
        for (int64_t r = r0; r < r1; ++r)
            for (int64_t c = c0; c < c1; ++c) {
                float v = (float)(unit_value((uint64_t)(r * cols + c), k0, k1, c8) * sigma);
                float x = v / s;
                x = fminf(fmaxf(x, -448.0f), 448.0f);
                q[r * cols + c] = f32_to_e4m3_rne(x);
            }
    }
}
