/*
 * Seeded synthetic inputs for the weight-only NVFP4 GEMV.
 *
 * This module only MANUFACTURES inputs: normal draws, their bf16 rounding and
 * the NVFP4 quantisation recipe that turns fp32 weights into stored bytes.
 * It holds none of the GEMV arithmetic (no decode of stored codes, no dot
 * products); the CPU oracle and the CUDA library both consume the bytes it
 * writes and neither shares code with it or with each other.
 *
 * Random stream: the splitmix64 generator (Steele, Lea, Flood, "Fast
 * splittable pseudorandom number generators", OOPSLA 2014), used in its
 * counter form so that draw i is mix(seed + (i + 1) * GAMMA) -- identical to
 * the i-th output of the sequential generator seeded with `seed`, but
 * computable for any i, which lets the draws be produced in parallel.
 * Uniforms in (0, 1] take the top 53 bits; normals come from the Box-Muller
 * transform on draw pairs (2j, 2j+1), both outputs used.
 *
 * Quantisation recipe (weights fp32 ~ N(0, sigma) -> NVFP4):
 *   global g   = amax|W| / (6 * 448)                       (fp32)
 *   group code = E4M3_RNE((amax_group / 6) / g)             (fp32 math, saturating at 448)
 *   element    = E2M1_RNE(w / (E4M3(code) * g))             (fp32 math, ties to even mantissa,
 *                                                            |.| > 6 saturates, sign kept)
 *   packing    = byte b of row n holds k = 2b in bits 0-3, k = 2b+1 in bits 4-7;
 *                scales row-major [N][K/16].
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* draw i of the stream seeded with `seed` */
static inline uint64_t draw(uint64_t seed, uint64_t i) { return mix64(seed + (i + 1) * GAMMA); }

/* uniform in (0, 1] from the top 53 bits */
static inline double unit(uint64_t z) { return (double)((z >> 11) + 1) * (1.0 / 9007199254740992.0); }

uint64_t synth_draw(uint64_t seed, uint64_t i) { return draw(seed, i); }

/* Normal draws number offset .. offset+count-1 (offset must be even: pairs start on even draws),
 * scaled by sigma, written as double. */
static void normals(uint64_t seed, uint64_t offset, int64_t count, double sigma, double* out) {
    const double two_pi = 6.283185307179586476925286766559;
    int64_t pairs = (count + 1) / 2;
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < pairs; ++j) {
        double u1 = unit(draw(seed, offset + 2 * (uint64_t)j));
        double u2 = unit(draw(seed, offset + 2 * (uint64_t)j + 1));
        double r = sqrt(-2.0 * log(u1));
        double t = two_pi * u2;
        out[2 * j] = sigma * r * cos(t);
        if (2 * j + 1 < count) out[2 * j + 1] = sigma * r * sin(t);
    }
}

int synth_normal_f64(uint64_t seed, uint64_t offset, int64_t count, double sigma, double* out) {
    if ((offset & 1) || count < 0 || (!out && count)) return -1;
    normals(seed, offset, count, sigma, out);
    return 0;
}

int synth_normal_f32(uint64_t seed, uint64_t offset, int64_t count, double sigma, float* out) {
    if ((offset & 1) || count < 0 || (!out && count)) return -1;
    const int64_t CH = 1 << 22;
    double* tmp = (double*)malloc(sizeof(double) * (size_t)(count < CH ? (count ? count : 1) : CH));
    if (!tmp) return -2;
    for (int64_t s = 0; s < count; s += CH) {
        int64_t c = count - s < CH ? count - s : CH;
        normals(seed, offset + (uint64_t)s, c, sigma, tmp);
        #pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < c; ++i) out[s + i] = (float)tmp[i];
    }
    free(tmp);
    return 0;
}

/* fp32 -> bf16 bits, round to nearest even */
static inline uint16_t f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

uint16_t synth_f32_to_bf16(float f) { return f32_to_bf16(f); }

/* Normal draws (fp32 first, as the recipe states) rounded to bf16 bits. */
int synth_normal_bf16(uint64_t seed, uint64_t offset, int64_t count, double sigma, uint16_t* out) {
    if ((offset & 1) || count < 0 || (!out && count)) return -1;
    const int64_t CH = 1 << 22;
    double* tmp = (double*)malloc(sizeof(double) * (size_t)(count < CH ? (count ? count : 1) : CH));
    if (!tmp) return -2;
    for (int64_t s = 0; s < count; s += CH) {
        int64_t c = count - s < CH ? count - s : CH;
        normals(seed, offset + (uint64_t)s, c, sigma, tmp);
        #pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < c; ++i) out[s + i] = f32_to_bf16((float)tmp[i]);
    }
    free(tmp);
    return 0;
}

/* Round a positive finite value onto the E4M3 (FN variant: bias 7, max 448, no infinity)
 * grid, nearest-even, saturating at 448.  Returns the 8-bit code; *value gets the grid
 * value that code stands for (computed here from the rounding, not by decoding a code). */
static uint8_t e4m3_round(float vf, float* value) {
    double v = (double)vf;
    if (!(v > 0.0)) { *value = 0.0f; return 0; }
    if (v >= 448.0) { *value = 448.0f; return 0x7E; }
    int e;
    (void)frexp(v, &e);
    int E = e - 1; /* v in [2^E, 2^(E+1)) */
    if (E < -6) {
        /* below the smallest normal 2^-6: multiples of 2^-9 */
        double q = rint(ldexp(v, 9));
        *value = (float)ldexp(q, -9);
        return (uint8_t)q; /* q == 8 is the code of 2^-6 (exponent field 1, mantissa 0) */
    }
    double q = rint(ldexp(v, 3 - E)); /* 3 mantissa bits: q in [8, 16] */
    if (q == 16.0) { q = 8.0; E += 1; }
    *value = (float)ldexp(q, E - 3);
    return (uint8_t)(((E + 7) << 3) | ((int)q - 8));
}

/* Round onto the E2M1 grid {0, .5, 1, 1.5, 2, 3, 4, 6}, nearest with ties to the even
 * mantissa, saturating at 6; returns the 4-bit code with the sign in bit 3. */
static uint8_t e2m1_round(float r) {
    float a = fabsf(r);
    uint8_t c;
    if (a <= 0.25f) c = 0;
    else if (a < 0.75f) c = 1;
    else if (a <= 1.25f) c = 2;
    else if (a < 1.75f) c = 3;
    else if (a <= 2.5f) c = 4;
    else if (a < 3.5f) c = 5;
    else if (a <= 5.0f) c = 6;
    else c = 7;
    return (uint8_t)(c | (signbit(r) ? 8 : 0));
}

uint8_t synth_e4m3_round(float v, float* value) { return e4m3_round(v, value); }
uint8_t synth_e2m1_round(float r) { return e2m1_round(r); }

/* Quantise fp32 weights w[n][k] (k % 16 == 0) into packed nibbles [n][k/2] and
 * scale codes [n][k/16]; writes the fp32 global scale. */
int synth_quantize_nvfp4(const float* w, int64_t n, int64_t k, uint8_t* packed, uint8_t* scales,
                         float* global_scale) {
    if (n < 0 || k < 0 || (k % 16) || !global_scale) return -1;
    float amax = 0.0f;
    int64_t total = n * k;
    #pragma omp parallel for reduction(max : amax) schedule(static)
    for (int64_t i = 0; i < total; ++i) {
        float a = fabsf(w[i]);
        if (a > amax) amax = a;
    }
    float g = amax > 0.0f ? amax / (6.0f * 448.0f) : 1.0f;
    *global_scale = g;
    int64_t groups = k / 16;
    #pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < n; ++row) {
        const float* wr = w + row * k;
        for (int64_t gi = 0; gi < groups; ++gi) {
            const float* wg = wr + gi * 16;
            float ag = 0.0f;
            for (int j = 0; j < 16; ++j) {
                float a = fabsf(wg[j]);
                if (a > ag) ag = a;
            }
            float sv;
            float t = ag / 6.0f;
            uint8_t code = e4m3_round(t / g, &sv);
            scales[row * groups + gi] = code;
            float d = sv * g;
            for (int j = 0; j < 16; j += 2) {
                uint8_t lo = 0, hi = 0;
                if (d != 0.0f) {
                    lo = e2m1_round(wg[j] / d);
                    hi = e2m1_round(wg[j + 1] / d);
                }
                packed[row * (k / 2) + gi * 8 + j / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
    return 0;
}
