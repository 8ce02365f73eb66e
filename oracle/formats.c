/*
 * Oracle number formats: E2M1 (FP4), E8M0 scales, E4M3 (FP8), MXFP4 and MXFP8
 * blocks, the Q2_K-style 2-bit super-block, binary16 and bfloat16 rounding.
 *
 * TEST INFRASTRUCTURE (see oracle.h). Plain and slow on purpose.
 *
 * The pages name the formats without defining them: MXFP4 keeps the released
 * routed-expert weights ("DwarfStar", hysenlabs.com, "Model support and
 * quantisation"); the 2-bit build uses Q2_K for the routed down projection
 * ("DS4", dibi8.com, "Key architectural innovations" item 1). The element and
 * scale encodings below follow the OCP Microscaling Formats (MX) v1.0
 * specification: E2M1 with exponent bias 1, E4M3 with bias 7, E8M0 = 2^(e-127),
 * 32-element blocks whose shared scale is 2^(floor(log2(amax)) - emax_elem).
 * Readings where the pages and the spec leave a choice open:
 *  - an all-zero block gets scale byte 127 and all-zero codes;
 *  - elements round to nearest, ties to even mantissa, and saturate at the
 *    largest finite magnitude (6 for E2M1, 448 for E4M3);
 *  - the sign bit is kept, so -0.0 and negatives that round to zero encode
 *    as the negative-zero code;
 *  - the Q2_K-style super-block's byte layout and its min-max encoder are this
 *    project's own (no GGUF compatibility is claimed).
 */
#include <math.h>
#include <string.h>

#include "oracle.h"

/* ---- element formats ------------------------------------------------------ */

int ora_floor_log2(double a) {
    int ex;
    frexp(a, &ex); /* a = f * 2^ex with f in [0.5, 1) */
    return ex - 1;
}

double ora_e2m1_value(uint8_t code) {
    const int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    const double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

double ora_e8m0_value(uint8_t e) { return e == 0xFF ? NAN : ldexp(1.0, (int)e - 127); }

double ora_e4m3_value(uint8_t code) {
    const int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    const double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* E2M1 magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6 (codes 0..7). Rounding to
 * nearest with ties to the even mantissa puts the tie points 0.25, 1.25, 2.5
 * and 5 on the lower neighbour and 0.75, 1.75, 3.5 on the upper one. */
uint8_t ora_e2m1_encode(double y) {
    const uint8_t s = signbit(y) ? 8 : 0;
    const double a = fabs(y);
    uint8_t m;
    if (a <= 0.25) m = 0;
    else if (a < 0.75) m = 1;
    else if (a <= 1.25) m = 2;
    else if (a < 1.75) m = 3;
    else if (a <= 2.5) m = 4;
    else if (a < 3.5) m = 5;
    else if (a <= 5.0) m = 6;
    else m = 7;
    return s | m;
}

uint8_t ora_e2m1_encode_nearest(double y) {
    const uint8_t s = signbit(y) ? 8 : 0;
    const double a = fabs(y);
    if (a >= 6.0) return s | 7; /* beyond the largest magnitude: saturate */
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c < 8; ++c) {
        const double dist = fabs(a - ora_e2m1_value((uint8_t)c));
        if (dist < bd || (dist == bd && (c & 1) == 0)) {
            bd = dist;
            best = c;
        }
    }
    return s | (uint8_t)best;
}

uint8_t ora_e4m3_encode(double y) {
    const uint8_t s = signbit(y) ? 0x80 : 0;
    const double a = fabs(y);
    if (a >= 448.0) return s | 0x7E;
    if (a == 0.0) return s;
    const int k = ora_floor_log2(a);
    const double ulp = (k < -6) ? ldexp(1.0, -9) : ldexp(1.0, k - 3);
    const double v = nearbyint(a / ulp) * ulp; /* default rounding: nearest, ties to even */
    if (v == 0.0) return s;
    if (v < ldexp(1.0, -6)) return s | (uint8_t)(v / ldexp(1.0, -9));
    const int k2 = ora_floor_log2(v);
    const int e = k2 + 7;
    const int m = (int)(ldexp(v, -k2) * 8.0) - 8;
    return s | (uint8_t)(e << 3) | (uint8_t)m;
}

uint8_t ora_e4m3_encode_nearest(double y) {
    const uint8_t s = signbit(y) ? 0x80 : 0;
    const double a = fabs(y);
    if (a >= 448.0) return s | 0x7E; /* beyond the largest magnitude: saturate */
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c < 0x7F; ++c) { /* 0x7F is NaN */
        const double dist = fabs(a - ora_e4m3_value((uint8_t)c));
        if (dist < bd || (dist == bd && (c & 1) == 0)) {
            bd = dist;
            best = c;
        }
    }
    return s | (uint8_t)best;
}

/* ---- binary16 / bfloat16 ---------------------------------------------------- */

uint16_t ora_f32_to_f16(float f) {
    const double v = f;
    const uint16_t s = signbit(v) ? 0x8000 : 0;
    if (isnan(v)) return 0x7E00;
    const double a = fabs(v);
    if (a == 0.0) return s;
    if (isinf(a)) return s | 0x7C00;
    const int k = ora_floor_log2(a);
    const double ulp = (k < -14) ? ldexp(1.0, -24) : ldexp(1.0, k - 10);
    const double r = nearbyint(a / ulp) * ulp;
    if (r > 65504.0) return s | 0x7C00;
    if (r == 0.0) return s;
    if (r < ldexp(1.0, -14)) return s | (uint16_t)(r / ldexp(1.0, -24));
    const int k2 = ora_floor_log2(r);
    return s | (uint16_t)((k2 + 15) << 10) | (uint16_t)(ldexp(r, -k2) * 1024.0 - 1024.0);
}

double ora_f16_value(uint16_t h) {
    const int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
    double mag;
    if (e == 31) mag = m ? NAN : INFINITY;
    else if (e == 0) mag = ldexp((double)m, -24);
    else mag = ldexp(1.0 + m / 1024.0, e - 15);
    return s ? -mag : mag;
}

uint16_t ora_f64_to_bf16(double v) {
    const uint16_t s = signbit(v) ? 0x8000 : 0;
    if (isnan(v)) return 0x7FC0;
    const double a = fabs(v);
    if (a == 0.0) return s;
    if (isinf(a)) return s | 0x7F80;
    const int k = ora_floor_log2(a);
    const double ulp = (k < -126) ? ldexp(1.0, -133) : ldexp(1.0, k - 7);
    const double r = nearbyint(a / ulp) * ulp;
    if (r > ldexp(2.0 - ldexp(1.0, -7), 127)) return s | 0x7F80;
    if (r == 0.0) return s;
    if (r < ldexp(1.0, -126)) return s | (uint16_t)(r / ldexp(1.0, -133));
    const int k2 = ora_floor_log2(r);
    return s | (uint16_t)((k2 + 127) << 7) | (uint16_t)(ldexp(r, -k2) * 128.0 - 128.0);
}

double ora_bf16_value(uint16_t b) {
    const uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ---- MX blocks ------------------------------------------------------------- */

/* Shared scale exponent of a block with largest magnitude amax > 0, clamped
 * to the E8M0 range. emax_elem is 2 for E2M1 and 8 for E4M3. */
static int mx_shared_exp(double amax, int emax_elem) {
    int se = ora_floor_log2(amax) - emax_elem;
    if (se < -127) se = -127;
    if (se > 127) se = 127;
    return se;
}

/* One MXFP4 block of 32 values: 16 code bytes (element 2i in the low
 * nibble) and the E8M0 scale byte. */
static uint8_t mxfp4_block(const double *v, uint8_t *c) {
    double amax = 0.0;
    for (int i = 0; i < 32; ++i) amax = fmax(amax, fabs(v[i]));
    if (amax == 0.0) {
        memset(c, 0, 16);
        return 127;
    }
    const int se = mx_shared_exp(amax, 2);
    for (int i = 0; i < 32; i += 2) {
        const uint8_t lo = ora_e2m1_encode(ldexp(v[i], -se));
        const uint8_t hi = ora_e2m1_encode(ldexp(v[i + 1], -se));
        c[i / 2] = (uint8_t)(lo | (hi << 4));
    }
    return (uint8_t)(se + 127);
}

void ora_mxfp4_quantize(const float *w, int64_t rows, int64_t K, uint8_t *codes, uint8_t *scales) {
    const int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double buf[32];
        for (int64_t b = 0; b < nb; ++b) {
            for (int i = 0; i < 32; ++i) buf[i] = (double)w[r * K + b * 32 + i];
            scales[r * nb + b] = mxfp4_block(buf, codes + r * (K / 2) + b * 16);
        }
    }
}

void ora_mxfp4_quantize_f64(const double *v, int64_t rows, int64_t K, uint8_t *codes, uint8_t *scales) {
    const int64_t nb = K / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nb; ++b)
            scales[r * nb + b] = mxfp4_block(v + r * K + b * 32, codes + r * (K / 2) + b * 16);
}

void ora_mxfp4_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t K,
                          float *out) {
    const int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t i = 0; i < K; ++i) {
            const uint8_t byte = codes[r * (K / 2) + i / 2];
            const uint8_t code = (i & 1) ? (byte >> 4) : (byte & 15);
            out[r * K + i] = (float)(ora_e2m1_value(code) * ora_e8m0_value(scales[r * nb + i / 32]));
        }
}

void ora_mxfp8_quantize_f64(const double *v, int64_t rows, int64_t K, uint8_t *codes,
                            uint8_t *scales) {
    const int64_t nb = K / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nb; ++b) {
            const double *x = v + r * K + b * 32;
            uint8_t *c = codes + r * K + b * 32;
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) amax = fmax(amax, fabs(x[i]));
            if (amax == 0.0) {
                scales[r * nb + b] = 127;
                memset(c, 0, 32);
                continue;
            }
            const int se = mx_shared_exp(amax, 8);
            scales[r * nb + b] = (uint8_t)(se + 127);
            for (int i = 0; i < 32; ++i) c[i] = ora_e4m3_encode(ldexp(x[i], -se));
        }
}

void ora_mxfp8_quantize_bf16(const uint16_t *x, int64_t rows, int64_t K, uint8_t *codes,
                             uint8_t *scales) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double buf[32];
        for (int64_t b = 0; b < K / 32; ++b) {
            for (int i = 0; i < 32; ++i) buf[i] = ora_bf16_value(x[r * K + b * 32 + i]);
            /* one 32-element block at a time through the fp64 encoder */
            uint8_t sc;
            ora_mxfp8_quantize_f64(buf, 1, 32, codes + r * K + b * 32, &sc);
            scales[r * (K / 32) + b] = sc;
        }
    }
}

void ora_mxfp8_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t K,
                          double *out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t i = 0; i < K; ++i)
            out[r * K + i] = ora_e4m3_value(codes[r * K + i]) * ora_e8m0_value(scales[r * (K / 32) + i / 32]);
}

/* ---- Q2_K-style super-block --------------------------------------------------
 * 256 weights: 16 sub-blocks of 16, each with a 4-bit scale sc and a 4-bit min m,
 * 2-bit quants q, and fp16 super-scales d and dmin:
 *     w = d * sc * q - dmin * m.
 * Bytes: [0,16) sc | m << 4 per sub-block; [16,80) quant n at byte 16 + n/4,
 * bits 2*(n%4); [80,82) d; [82,84) dmin (little-endian binary16).
 * Encoder (fp32 arithmetic, roundf = half away from zero):
 *     mn_i = max(0, -min w), rng_i = (max w + mn_i) / 3
 *     d = f16(max rng_i / 15), dmin = f16(max mn_i / 15)
 *     sc_i = clamp(round(rng_i / d), 0, 15), m_i = clamp(round(mn_i / dmin), 0, 15)
 *     q = clamp(round((w + dmin * m_i) / (d * sc_i)), 0, 3)
 * with 0 wherever the divisor is 0. */

static float clampf(float v, float lo, float hi) { return v < lo ? lo : (v > hi ? hi : v); }

static void q2k_encode_block(const float *w, uint8_t *blk) {
    float rng[16], mn[16], rmax = 0.0f, mmax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float lo = w[16 * i], hi = w[16 * i];
        for (int j = 1; j < 16; ++j) {
            lo = fminf(lo, w[16 * i + j]);
            hi = fmaxf(hi, w[16 * i + j]);
        }
        mn[i] = fmaxf(0.0f, -lo);
        rng[i] = (hi + mn[i]) / 3.0f;
        rmax = fmaxf(rmax, rng[i]);
        mmax = fmaxf(mmax, mn[i]);
    }
    const uint16_t dh = ora_f32_to_f16(rmax / 15.0f), mh = ora_f32_to_f16(mmax / 15.0f);
    const float d = (float)ora_f16_value(dh), dmin = (float)ora_f16_value(mh);
    memset(blk, 0, ORA_Q2K_BYTES);
    for (int i = 0; i < 16; ++i) {
        const int sc = d > 0.0f ? (int)clampf(roundf(rng[i] / d), 0.0f, 15.0f) : 0;
        const int m = dmin > 0.0f ? (int)clampf(roundf(mn[i] / dmin), 0.0f, 15.0f) : 0;
        blk[i] = (uint8_t)(sc | (m << 4));
        for (int j = 0; j < 16; ++j) {
            const int n = 16 * i + j;
            int q = 0;
            if (sc > 0) {
                const float num = w[n] + dmin * (float)m;
                q = (int)clampf(roundf(num / (d * (float)sc)), 0.0f, 3.0f);
            }
            blk[16 + n / 4] |= (uint8_t)(q << (2 * (n % 4)));
        }
    }
    blk[80] = (uint8_t)(dh & 0xFF);
    blk[81] = (uint8_t)(dh >> 8);
    blk[82] = (uint8_t)(mh & 0xFF);
    blk[83] = (uint8_t)(mh >> 8);
}

static void q2k_decode_block(const uint8_t *blk, float *w) {
    const float d = (float)ora_f16_value((uint16_t)(blk[80] | (blk[81] << 8)));
    const float dmin = (float)ora_f16_value((uint16_t)(blk[82] | (blk[83] << 8)));
    for (int n = 0; n < 256; ++n) {
        const int i = n / 16;
        const int sc = blk[i] & 15, m = blk[i] >> 4;
        const int q = (blk[16 + n / 4] >> (2 * (n % 4))) & 3;
        const float a = (d * (float)sc) * (float)q; /* exact: <= 11 + 4 + 2 bits */
        const float b = dmin * (float)m;            /* exact */
        w[n] = a - b;                               /* the only rounding */
    }
}

void ora_q2k_quantize(const float *w, int64_t rows, int64_t K, uint8_t *blocks) {
    const int64_t nb = K / ORA_Q2K_BLOCK;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nb; ++b)
            q2k_encode_block(w + r * K + b * ORA_Q2K_BLOCK, blocks + (r * nb + b) * ORA_Q2K_BYTES);
}

void ora_q2k_dequantize(const uint8_t *blocks, int64_t rows, int64_t K, float *out) {
    const int64_t nb = K / ORA_Q2K_BLOCK;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nb; ++b)
            q2k_decode_block(blocks + (r * nb + b) * ORA_Q2K_BYTES, out + r * K + b * ORA_Q2K_BLOCK);
}
