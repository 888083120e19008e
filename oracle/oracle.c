/*
 * oracle.c -- CPU oracle for weight-only quantized decode (TEST INFRASTRUCTURE
 * ONLY; see oracle.h for who may call it and for the page citations).
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -fopenmp -ffp-contract=off
 *        -fno-fast-math oracle.c -lm
 * FP contraction is off so that every fp32 operation below is one IEEE
 * operation rounded to nearest-even, as written.
 */
#include "oracle.h"

#include <math.h>
#include <omp.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- fp16 --- */

/* Round the non-negative integer m right by s bits, ties to even. */
static uint64_t shift_round_half_even(uint64_t m, int s) {
    if (s <= 0) return m << (-s);
    if (s >= 64) return 0;
    uint64_t q = m >> s;
    uint64_t r = m & ((((uint64_t)1) << s) - 1);
    uint64_t half = ((uint64_t)1) << (s - 1);
    if (r > half || (r == half && (q & 1))) q += 1;
    return q;
}

uint16_t orc_f32_to_f16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t e32 = (u >> 23) & 0xFFu;
    uint32_t m32 = u & 0x7FFFFFu;
    if (e32 == 0xFFu) /* Inf or NaN (NaN keeps a quiet payload bit) */
        return (uint16_t)(sign | 0x7C00u | (m32 ? 0x0200u : 0u));
    if (e32 == 0) /* zero or fp32 subnormal: |f| < 2^-126, far below 2^-25 */
        return sign;
    /* |f| = M * 2^(e32 - 150) with the 24-bit integer significand M. */
    uint64_t M = (uint64_t)(m32 | 0x800000u);
    int e16 = (int)e32 - 127 + 15; /* biased binary16 exponent if normal */
    if (e16 >= 1) {
        /* Normal range: keep 11 significant bits.  A carry out of the
         * significand (M16 == 2048) correctly bumps the exponent, and
         * e16 reaching 31 yields the Inf encoding. */
        uint64_t M16 = shift_round_half_even(M, 13);
        uint32_t h = ((uint32_t)e16 << 10) + (uint32_t)(M16 - 1024u);
        if (h >= 0x7C00u) return (uint16_t)(sign | 0x7C00u);
        return (uint16_t)(sign | h);
    }
    /* Subnormal range: value / 2^-24 = M * 2^(e32 - 126). */
    uint64_t M16 = shift_round_half_even(M, 126 - (int)e32);
    return (uint16_t)(sign | (uint32_t)M16); /* 1024 -> smallest normal */
}

double orc_f16_to_f64(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return sign ? -v : v;
}

float orc_f16_to_f32(uint16_t h) { return (float)orc_f16_to_f64(h); }

double orc_rint_half_even(float r) {
    double x = (double)r; /* exact */
    double fl = floor(x);
    double d = x - fl; /* exact: fl and x share the binade or fl == 0 */
    if (d > 0.5) return fl + 1.0;
    if (d < 0.5) return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* ------------------------------------------------ int8 per-block-32 ------ */

void orc_quantize_block32(const float* w, int64_t n, int64_t k, int8_t* codes,
                          uint16_t* scales) {
    const int64_t nb = k / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* wb = w + r * k + b * 32;
            /* absmax over the block of 32 consecutive inputs (no clipping) */
            float a = 0.0f;
            for (int j = 0; j < 32; ++j) {
                float v = fabsf(wb[j]);
                if (v > a) a = v;
            }
            /* scale = absmax / 127 in fp32, stored as fp16 (RNE) */
            volatile float t = a / 127.0f;
            uint16_t s16 = orc_f32_to_f16(t);
            scales[r * nb + b] = s16;
            float s = orc_f16_to_f32(s16);
            int8_t* qb = codes + r * k + b * 32;
            for (int j = 0; j < 32; ++j) {
                if (s == 0.0f) {
                    qb[j] = 0;
                    continue;
                }
                /* code = round-half-even(w / s) with the stored scale, fp32
                 * IEEE division, clamped to the symmetric range [-127, 127] */
                volatile float ratio = wb[j] / s;
                double q = orc_rint_half_even(ratio);
                if (q > 127.0) q = 127.0;
                if (q < -127.0) q = -127.0;
                qb[j] = (int8_t)q;
            }
        }
    }
}

/* ------------------------------------------------ int4 group-64 affine --- */

void orc_quantize_int4_g64(const float* w, int64_t n, int64_t k, uint8_t* codes,
                           uint16_t* scales, uint16_t* biases) {
    const int64_t ng = k / 64;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        for (int64_t g = 0; g < ng; ++g) {
            const float* wg = w + r * k + g * 64;
            float mx = wg[0], mn = wg[0];
            for (int j = 1; j < 64; ++j) {
                if (wg[j] > mx) mx = wg[j];
                if (wg[j] < mn) mn = wg[j];
            }
            /* a signed-zero extreme counts as +0 (x + 0 maps -0 to +0 and
             * leaves every other value unchanged) */
            volatile float zero = 0.0f;
            mx = mx + zero;
            mn = mn + zero;
            /* scale = (max - min) / 15 and bias = min, both fp16 (RNE);
             * each fp32 operation rounded on its own */
            volatile float range = mx - mn;
            volatile float t = range / 15.0f;
            uint16_t s16 = orc_f32_to_f16(t);
            uint16_t b16 = orc_f32_to_f16(mn);
            scales[r * ng + g] = s16;
            biases[r * ng + g] = b16;
            float s = orc_f16_to_f32(s16);
            float bias = orc_f16_to_f32(b16);
            uint8_t q[64];
            for (int j = 0; j < 64; ++j) {
                if (s == 0.0f) {
                    q[j] = 0;
                    continue;
                }
                volatile float centred = wg[j] - bias;
                volatile float ratio = centred / s;
                double v = orc_rint_half_even(ratio);
                if (v > 15.0) v = 15.0;
                if (v < 0.0) v = 0.0;
                q[j] = (uint8_t)v;
            }
            /* two codes per byte, the even k in the low nibble */
            uint8_t* cg = codes + r * (k / 2) + g * 32;
            for (int j = 0; j < 32; ++j)
                cg[j] = (uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));
        }
    }
}

/* ------------------------------------------------------------ dequant --- */

void orc_dequant_row_i8(const int8_t* codes, const uint16_t* scales, int64_t k,
                        int64_t r, double* out) {
    for (int64_t j = 0; j < k; ++j) {
        double s = orc_f16_to_f64(scales[r * (k / 32) + j / 32]);
        out[j] = (double)codes[r * k + j] * s;
    }
}

void orc_dequant_row_i4(const uint8_t* codes, const uint16_t* scales,
                        const uint16_t* biases, int64_t k, int64_t r,
                        double* out) {
    for (int64_t j = 0; j < k; ++j) {
        uint8_t byte = codes[r * (k / 2) + j / 2];
        int q = (j & 1) ? (byte >> 4) : (byte & 0x0F);
        double s = orc_f16_to_f64(scales[r * (k / 64) + j / 64]);
        double b = orc_f16_to_f64(biases[r * (k / 64) + j / 64]);
        out[j] = (double)q * s + b;
    }
}

/* ------------------------------------------------------------- matvec --- */

void orc_matvec(int fmt, const void* codes, const uint16_t* scales,
                const uint16_t* biases, int64_t n, int64_t k, const uint16_t* x,
                double* y, double* mag) {
    /* x and the per-row side data are converted to fp64 once (exact); the
     * sums run in index order. */
    double* xd = (double*)malloc(sizeof(double) * (size_t)k);
    for (int64_t j = 0; j < k; ++j) xd[j] = orc_f16_to_f64(x[j]);
    const int64_t blk = fmt == 0 ? 32 : 64;
    const int64_t nb = fmt == 2 ? 0 : k / blk;
#pragma omp parallel
    {
        double* sd = (double*)malloc(sizeof(double) * (size_t)(nb > 0 ? nb : 1));
        double* bd = (double*)malloc(sizeof(double) * (size_t)(nb > 0 ? nb : 1));
#pragma omp for schedule(static)
        for (int64_t r = 0; r < n; ++r) {
            for (int64_t b = 0; b < nb; ++b) {
                sd[b] = orc_f16_to_f64(scales[r * nb + b]);
                bd[b] = fmt == 0 ? 0.0 : orc_f16_to_f64(biases[r * nb + b]);
            }
            double acc = 0.0, am = 0.0;
            for (int64_t j = 0; j < k; ++j) {
                double wdq;
                if (fmt == 2) {
                    const uint16_t* c = (const uint16_t*)codes;
                    wdq = orc_f16_to_f64(c[r * k + j]);
                } else if (fmt == 0) {
                    const int8_t* c = (const int8_t*)codes;
                    wdq = (double)c[r * k + j] * sd[j / 32];
                } else {
                    const uint8_t* c = (const uint8_t*)codes;
                    uint8_t byte = c[r * (k / 2) + j / 2];
                    int q = (j & 1) ? (byte >> 4) : (byte & 0x0F);
                    wdq = (double)q * sd[j / 64] + bd[j / 64];
                }
                double p = wdq * xd[j];
                acc += p;
                am += fabs(p);
            }
            if (y) y[r] = acc;
            if (mag) mag[r] = am;
        }
        free(sd);
        free(bd);
    }
    free(xd);
}

/* ----------------------------------------------------- fp64 -> fp16 --- */

uint16_t orc_f64_to_f16(double d) {
    uint16_t sign = signbit(d) ? 0x8000u : 0u;
    double a = fabs(d);
    if (isnan(d)) return (uint16_t)(sign | 0x7E00u);
    if (isinf(a)) return (uint16_t)(sign | 0x7C00u);
    if (a == 0.0) return sign;
    int e2;
    frexp(a, &e2);       /* a = m * 2^e2, 0.5 <= m < 1, so 2^(e2-1) <= a < 2^e2 */
    int E = e2 - 1;      /* unbiased exponent of a */
    if (E < -14) E = -14; /* subnormal range: fixed quantum 2^-24 */
    /* the significand in units of the quantum 2^(E-10) (exact power-of-two
     * scaling), rounded half to even */
    double q = nearbyint(ldexp(a, 10 - E));
    if (q >= 2048.0) { /* rounded up to the next binade */
        q /= 2.0;
        E += 1;
    }
    if (E > 15) return (uint16_t)(sign | 0x7C00u);
    if (q < 1024.0) return (uint16_t)(sign | (uint16_t)q); /* subnormal (E == -14) */
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | ((uint16_t)q & 0x3FFu));
}

/* ------------------------------------------------------------ RMSNorm --- */

void orc_rmsnorm(const float* h, const uint16_t* gamma, int64_t k, double eps, uint16_t* x,
                 double* x_exact) {
    double ss = 0.0;
    for (int64_t i = 0; i < k; ++i) ss += (double)h[i] * (double)h[i];
    const double rms = sqrt(ss / (double)k + eps);
    for (int64_t i = 0; i < k; ++i) {
        const double v = (double)h[i] * orc_f16_to_f64(gamma[i]) / rms;
        if (x_exact) x_exact[i] = v;
        x[i] = orc_f64_to_f16(v);
    }
}

/* --------------------------------------------------- decode attention --- */

void orc_rope(const double* x, int64_t d, int64_t pos, double theta, double* out) {
    const int64_t half = d / 2;
    for (int64_t i = 0; i < half; ++i) {
        const double f = pow(theta, -2.0 * (double)i / (double)d);
        const double a = (double)pos * f;
        const double c = cos(a), s = sin(a);
        out[i] = x[i] * c - x[i + half] * s;
        out[i + half] = x[i + half] * c + x[i] * s;
    }
}

void orc_decode_attention(const float* qkv, int64_t hq, int64_t hkv, int64_t d,
                          const uint16_t* kcache, const uint16_t* vcache, int64_t l_max,
                          int64_t pos, double theta, uint16_t* k_new, uint16_t* v_new,
                          double* o, double* mag) {
    const int64_t group = hq / hkv;
    const double scale = 1.0 / sqrt((double)d);
    double* xin = (double*)malloc((size_t)d * sizeof(double));
    double* rot = (double*)malloc((size_t)d * sizeof(double));
    double* kj = (double*)malloc((size_t)d * sizeof(double));
    double* s = (double*)malloc((size_t)(pos + 1) * sizeof(double));
    /* the appended rows */
    for (int64_t g = 0; g < hkv; ++g) {
        for (int64_t i = 0; i < d; ++i) xin[i] = (double)qkv[hq * d + g * d + i];
        orc_rope(xin, d, pos, theta, rot);
        for (int64_t i = 0; i < d; ++i) {
            k_new[g * d + i] = orc_f64_to_f16(rot[i]);
            v_new[g * d + i] = orc_f64_to_f16((double)qkv[hq * d + hkv * d + g * d + i]);
        }
    }
    for (int64_t h = 0; h < hq; ++h) {
        const int64_t g = h / group;
        for (int64_t i = 0; i < d; ++i) xin[i] = (double)qkv[h * d + i];
        orc_rope(xin, d, pos, theta, rot);
        double m = -HUGE_VAL;
        for (int64_t j = 0; j <= pos; ++j) {
            for (int64_t i = 0; i < d; ++i)
                kj[i] = orc_f16_to_f64(j == pos ? k_new[g * d + i]
                                                : kcache[(g * l_max + j) * d + i]);
            double dot = 0.0;
            for (int64_t i = 0; i < d; ++i) dot += rot[i] * kj[i];
            s[j] = dot * scale;
            if (s[j] > m) m = s[j];
        }
        double z = 0.0;
        for (int64_t j = 0; j <= pos; ++j) {
            s[j] = exp(s[j] - m);
            z += s[j];
        }
        for (int64_t i = 0; i < d; ++i) {
            double acc = 0.0, mg = 0.0;
            for (int64_t j = 0; j <= pos; ++j) {
                const double v = orc_f16_to_f64(j == pos ? v_new[g * d + i]
                                                         : vcache[(g * l_max + j) * d + i]);
                const double p = s[j] / z;
                acc += p * v;
                mg += p * fabs(v);
            }
            o[h * d + i] = acc;
            mag[h * d + i] = mg;
        }
    }
    free(xin);
    free(rot);
    free(kj);
    free(s);
}

/* ------------------------------------------------------------- SwiGLU --- */

double orc_silu(double g) { return g / (1.0 + exp(-g)); }

double orc_silu_grad(double g) {
    double sig = 1.0 / (1.0 + exp(-g));
    return sig * (1.0 + g * (1.0 - sig));
}

double orc_ulp_f16(double v) {
    v = fabs(v);
    if (v < ldexp(1.0, -14)) return ldexp(1.0, -24);
    int e;
    frexp(v, &e); /* v = f * 2^e with f in [0.5, 1) */
    return ldexp(1.0, (e - 1) - 10);
}

void orc_swiglu(const double* g, const double* u, const double* mag_g,
                const double* mag_u, int64_t n, double tol, double* h,
                double* bound) {
    for (int64_t i = 0; i < n; ++i) {
        double sg = orc_silu(g[i]);
        h[i] = sg * u[i];
        if (bound) {
            double e = tol * (fabs(orc_silu_grad(g[i])) * mag_g[i] * fabs(u[i]) +
                              fabs(sg) * mag_u[i]);
            bound[i] = e + 0.5 * orc_ulp_f16(fabs(h[i]) + e);
        }
    }
}

/* ------------------------------------------------------------- argmax --- */

int64_t orc_argmax(const double* v, int64_t n) {
    int64_t best = 0;
    for (int64_t i = 1; i < n; ++i)
        if (v[i] > v[best]) best = i;
    return best;
}

/* ------------------------------------------------------------ threads --- */

int orc_num_threads(void) { return omp_get_max_threads(); }

/* Threads the parallel loops above use from now on (the baseline timing runs
 * the oracle once on one thread and once on every core). */
void orc_set_num_threads(int n) { omp_set_num_threads(n > 0 ? n : 1); }
