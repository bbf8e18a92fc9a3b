/*
 * CPU ORACLE for the weight-only NVFP4 GEMV -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may load this
 * library.  The product path (the CUDA library) never calls it and shares no code,
 * header, table or constant with it.
 *
 * What it computes (the plain definition of the operation, no blocking or reordering):
 *
 *   y[m][n] = sum_{k=0}^{K-1} E2M1(nib(n,k)) * E4M3(S[n][k/16]) * g * x[m][k]
 *
 * summed in fp64 in increasing k; every term is exact in fp64 (2 x 4 x 24 x 8 significant
 * bits), so y differs from the real-number result only by the fp64 rounding of the sum.
 * A[m][n] = sum_k |term| is returned beside it as the tolerance scale.
 * Source: the weight-only 4-bit GEMV family "w4a16_gemv" / "w4a16_gemv_dual" with weights
 * "nvfp4/g16" and bf16 activations ("Blueprint - circuit executor" page for
 * qwen3.8-27b-nvfp4 on GB10, tables "Kernels the plan launches" and "Weighted nodes"),
 * and the practice of an fp64 reference per projection class (TensorFold issue #603,
 * "Port Qwen3.8-27B ... to the native CUDA engine", maintainers' reply).
 *
 * The fused dual:  o[m][n] = silu(yg[m][n]) * yu[m][n],  silu(t) = t / (1 + exp(-t)),
 * all in fp64 (the SiLU(gate)*up of the SwiGLU FFN that the GB10 plan runs as
 * w4a16_gemv_dual_sw followed by moe_silu_mul).
 *
 * Input prologues (the GEMV's neighbours in the decode step: "residual_add_rms_norm",
 * "rms_norm" and "sigmoid_gate_mul" in the same page's table "Kernels the plan launches"; the
 * pages list them by name, the formulas are the standard RMS normalisation with a gain and
 * the sigmoid output gate of gated attention):
 *   add + RMS norm:  h = bf16(x + r);  xn = bf16(h * gamma / sqrt(mean_k(h^2) + eps))
 *   sigmoid gate:    xo = bf16(a * sigmoid(gate)),  sigmoid(t) = 1 / (1 + exp(-t))
 *   gated RMS norm ("gated_rms_norm_f32_input", the GatedDeltaNet's output norm before its
 *   output projection): x in fp32, normalised per group of G channels (one head),
 *                    xo = bf16(x * gamma[k mod G] * silu(z) / sqrt(mean_group(x^2) + eps)),
 *                    silu(t) = t / (1 + exp(-t))
 * in fp64 with one rounding to bf16 at the end of each line.
 *
 * Formats, written from their definitions (the pages name the format, not its bits):
 *   E2M1 nibble: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0;
 *                exponent 0 is subnormal: 0.5 * m.
 *   E4M3 byte (OCP 8-bit FP, "FN" variant): sign bit 7, exponent bits 6..3 (bias 7),
 *                mantissa bits 2..0; exponent 0 is subnormal m * 2^-9; 0x7F / 0xFF are NaN;
 *                no infinities; largest finite 448.
 *   Packing: byte b of row n holds k = 2b in bits 0..3 and k = 2b+1 in bits 4..7;
 *            scales row-major [N][K/16]; x bf16 row-major with row stride ldx.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <omp.h>

double oracle_e2m1(uint8_t nib) {
    int s = (nib >> 3) & 1, e = (nib >> 1) & 3, m = nib & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

double oracle_e4m3(uint8_t c) {
    int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* bf16 bit pattern -> value */
double oracle_bf16_value(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* fp64 -> bf16 bits, round to nearest even, taken directly from the double (no pass
 * through fp32, so there is one rounding).  bf16: 8 significant bits, exponent range
 * as fp32, subnormal quantum 2^-133, overflow to infinity. */
uint16_t oracle_bf16_rne(double d) {
    if (isnan(d)) return 0x7FC0;
    uint16_t sign = signbit(d) ? 0x8000 : 0;
    double a = fabs(d);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7F80;
    int e;
    (void)frexp(a, &e);            /* a in [2^(e-1), 2^e) */
    int qexp = e - 8;              /* 8 significant bits */
    if (qexp < -133) qexp = -133;  /* subnormal quantum */
    double q = rint(ldexp(a, -qexp)) ;  /* nearest-even on the grid */
    double r = ldexp(q, qexp);
    /* largest finite bf16 is (2 - 2^-7) * 2^127; anything that rounds above it is inf */
    if (r > ldexp(255.0, 120)) return sign | 0x7F80;
    float f = (float)r;            /* exact: r is on the bf16 grid */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)((u >> 16) & 0x7FFF);
}

static double T2[16], T4[256];
static int tables_ready = 0;

static void tables(void) {
    if (tables_ready) return;
    for (int i = 0; i < 16; ++i) T2[i] = oracle_e2m1((uint8_t)i);
    for (int i = 0; i < 256; ++i) T4[i] = oracle_e4m3((uint8_t)i);
    tables_ready = 1;
}

static int bad_args(const uint8_t* w, const uint8_t* s, const uint16_t* x, int64_t ldx, int m,
                    int64_t n, int64_t k) {
    if (m < 0 || n < 0 || k < 0 || (k % 16)) return 1;
    if (m > 0 && ldx < k) return 1;
    if (m > 0 && n > 0 && k > 0 && (!w || !s || !x)) return 1;
    return 0;
}

/* y and absum: [m][count] fp64, where count = n if rows == NULL, else the outputs listed
 * in rows[0..count).  threads <= 0 uses the OpenMP default. */
int oracle_gemv(const uint8_t* w, const uint8_t* s, float g, const uint16_t* x, int64_t ldx,
                int m, int64_t n, int64_t k, const int64_t* rows, int64_t count, double* y,
                double* absum, int threads) {
    if (bad_args(w, s, x, ldx, m, n, k)) return -1;
    if (!rows) count = n;
    tables();
    const double gd = (double)g;
    int nt = threads > 0 ? threads : omp_get_max_threads();
    #pragma omp parallel for schedule(dynamic, 4) num_threads(nt)
    for (int64_t j = 0; j < count; ++j) {
        int64_t row = rows ? rows[j] : j;
        const uint8_t* wr = w + row * (k / 2);
        const uint8_t* sr = s + row * (k / 16);
        for (int r = 0; r < m; ++r) {
            const uint16_t* xr = x + r * ldx;
            double acc = 0.0, aabs = 0.0;
            for (int64_t kk = 0; kk < k; ++kk) {
                uint8_t byte = wr[kk / 2];
                uint8_t nib = (kk & 1) ? (byte >> 4) : (byte & 15);
                double t = T2[nib] * T4[sr[kk / 16]] * gd * oracle_bf16_value(xr[kk]);
                acc += t;
                aabs += fabs(t);
            }
            y[r * count + j] = acc;
            if (absum) absum[r * count + j] = aabs;
        }
    }
    return 0;
}

/* o = silu(yg) * yu on the same x; yg and yu receive the two pre-activations,
 * ag and au (may be NULL) their sum_k |term|. */
int oracle_gemv_dual(const uint8_t* wg, const uint8_t* sg, float gg, const uint8_t* wu,
                     const uint8_t* su, float gu, const uint16_t* x, int64_t ldx, int m, int64_t n,
                     int64_t k, const int64_t* rows, int64_t count, double* o, double* yg,
                     double* yu, double* ag, double* au, int threads) {
    if (!rows) count = n;
    if (!o || !yg || !yu) return -1;
    if (oracle_gemv(wg, sg, gg, x, ldx, m, n, k, rows, count, yg, ag, threads)) return -1;
    if (oracle_gemv(wu, su, gu, x, ldx, m, n, k, rows, count, yu, au, threads)) return -1;
    for (int64_t i = 0; i < (int64_t)m * count; ++i) {
        double t = yg[i];
        o[i] = t / (1.0 + exp(-t)) * yu[i];
    }
    return 0;
}

/* ---------------------------------------------------------------------------------------- */
/* input prologues */

/* bf16 neighbours by ordinal (finite values; +0 and -0 share ordinal 0) */
static double bf16_step(uint16_t b, int dir) {
    int32_t o = (b & 0x8000) ? -(int32_t)(b & 0x7FFF) : (int32_t)(b & 0x7FFF);
    o += dir;
    uint16_t n = o < 0 ? (uint16_t)(0x8000 | (uint16_t)(-o)) : (uint16_t)o;
    return oracle_bf16_value(n);
}

/* 1 when v lies within a relative 2^-16 of a midpoint between bf16 neighbours, i.e. where an
 * evaluation less precise than fp64 may round the other way; 0 otherwise. */
static uint8_t near_midpoint(double v, uint16_t b) {
    if (v == 0.0 || (b & 0x7FFF) >= 0x7F80) return 0;
    double c = oracle_bf16_value(b);
    double lo = 0.5 * (c + bf16_step(b, -1)), hi = 0.5 * (c + bf16_step(b, +1));
    double d = fmin(fabs(v - lo), fabs(v - hi));
    return d <= ldexp(fabs(v), -16) ? 1 : 0;
}

/* Residual add, then RMS normalisation with a gain, row by row:
 *   h[m][k]  = bf16_rne(x[m][k] + r[m][k])     (the exact sum of two bf16 values, rounded once)
 *   ms[m]    = (1/K) sum_k h[m][k]^2           (fp64, increasing k)
 *   xn[m][k] = bf16_rne(h[m][k] * gamma[k] / sqrt(ms[m] + eps))
 * h is [m][k] (row stride k), xn likewise; near (may be NULL) marks xn elements whose fp64
 * value lies within a relative 2^-16 of a bf16 rounding midpoint. */
int oracle_add_rmsnorm(const uint16_t* x, int64_t ldx, const uint16_t* r, int64_t ldr,
                       const uint16_t* gamma, float eps, int m, int64_t k, uint16_t* h,
                       uint16_t* xn, uint8_t* near) {
    if (m < 0 || k <= 0 || ldx < k || ldr < k || !x || !r || !gamma || !h || !xn) return -1;
    if (!(eps >= 0.0f) || isinf(eps)) return -1;
    for (int i = 0; i < m; ++i) {
        double ss = 0.0;
        for (int64_t j = 0; j < k; ++j) {
            uint16_t hb = oracle_bf16_rne(oracle_bf16_value(x[i * ldx + j]) +
                                          oracle_bf16_value(r[i * ldr + j]));
            h[i * k + j] = hb;
            double hv = oracle_bf16_value(hb);
            ss += hv * hv;
        }
        double inv = 1.0 / sqrt(ss / (double)k + (double)eps);
        for (int64_t j = 0; j < k; ++j) {
            double v = oracle_bf16_value(h[i * k + j]) * oracle_bf16_value(gamma[j]) * inv;
            uint16_t b = oracle_bf16_rne(v);
            xn[i * k + j] = b;
            if (near) near[i * k + j] = near_midpoint(v, b);
        }
    }
    return 0;
}

/* xo[m][k] = bf16_rne(a[m][k] * sigmoid(gate[m][k])), sigmoid(t) = 1 / (1 + exp(-t)) in fp64;
 * xo is [m][k]; near as above. */
int oracle_sigmoid_gate(const uint16_t* a, int64_t lda, const uint16_t* gate, int64_t ldg, int m,
                        int64_t k, uint16_t* xo, uint8_t* near) {
    if (m < 0 || k <= 0 || lda < k || ldg < k || !a || !gate || !xo) return -1;
    for (int i = 0; i < m; ++i)
        for (int64_t j = 0; j < k; ++j) {
            double t = oracle_bf16_value(gate[i * ldg + j]);
            double v = oracle_bf16_value(a[i * lda + j]) * (1.0 / (1.0 + exp(-t)));
            uint16_t b = oracle_bf16_rne(v);
            xo[i * k + j] = b;
            if (near) near[i * k + j] = near_midpoint(v, b);
        }
    return 0;
}

/* Gated RMS norm over groups of `group` channels: for row i and group q (channels q*group ..),
 *   ms = (1/group) sum x^2 over the group (fp64, increasing k)
 *   xo[i][k] = bf16_rne(x[i][k] * gamma[k % group] * silu(z[i][k]) / sqrt(ms + eps))
 * x is fp32 [m][ldx], z bf16 [m][ldz], gamma bf16 [group]; xo is [m][k]; near as above. */
int oracle_gated_rmsnorm(const float* x, int64_t ldx, const uint16_t* z, int64_t ldz,
                         const uint16_t* gamma, int group, float eps, int m, int64_t k,
                         uint16_t* xo, uint8_t* near) {
    if (m < 0 || k <= 0 || group <= 0 || (k % group) || ldx < k || ldz < k || !x || !z ||
        !gamma || !xo)
        return -1;
    if (!(eps >= 0.0f) || isinf(eps)) return -1;
    for (int i = 0; i < m; ++i)
        for (int64_t q0 = 0; q0 < k; q0 += group) {
            double ss = 0.0;
            for (int j = 0; j < group; ++j) {
                double v = (double)x[i * ldx + q0 + j];
                ss += v * v;
            }
            double inv = 1.0 / sqrt(ss / (double)group + (double)eps);
            for (int j = 0; j < group; ++j) {
                double t = oracle_bf16_value(z[i * ldz + q0 + j]);
                double silu = t / (1.0 + exp(-t));
                double v = (double)x[i * ldx + q0 + j] * oracle_bf16_value(gamma[j]) * silu * inv;
                uint16_t b = oracle_bf16_rne(v);
                xo[i * k + q0 + j] = b;
                if (near) near[i * k + q0 + j] = near_midpoint(v, b);
            }
        }
    return 0;
}
