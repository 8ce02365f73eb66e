/*
 * Oracle expert FFN, shared expert, combine and the whole layer.
 *
 * TEST INFRASTRUCTURE (see oracle.h).
 *
 * The layer is DeepSeek V4 Flash's sparse MoE FFN (284B total / 13B active,
 * "DeepSeek V4 Flash ... on a Mac", grapeot.me, opening section): each token
 * goes through k routed experts, quantised, and an unquantised shared expert
 * ("DS4", dibi8.com, "Key architectural innovations" item 1). Every expert is a
 * SwiGLU FFN:
 *     g = W1 a,  u = W3 a,  h = silu(g) * u,  o = W2 h,  silu(g) = g / (1 + e^-g)
 * with W1, W3 of shape [F][d] and W2 of shape [d][F], blocks running along the
 * input dimension. The layer output is
 *     y[t] = sum_{j ascending} w[t,j] * o_{e(t,j)}[t]  (+ shared expert s[t]).
 * Readings (the pages are silent):
 *  - bf16-activation mode ("w4a16"): a = x (bf16) and h is rounded to bf16
 *    before W2; MXFP8 mode ("w4a8"): a is x quantised to MXFP8 along d and h
 *    is quantised to MXFP8 along F before W2; MXFP4 mode ("w4a4", both
 *    operands on the FP4 matrix instructions the pages name for Blackwell,
 *    "DwarfStar", hysenlabs.com, "Model support and quantisation"): the same
 *    with MXFP4 (E2M1 elements, the weights' rule);
 *  - the shared expert always takes bf16 x and rounds h to bf16; its gate is 1.
 * Arithmetic is fp64; MXFP4 dots sum each 32-element block, then apply the
 * block scale.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#include "oracle.h"

int ora_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads of later parallel regions (n >= 1); returns the count then in effect.
 * Threading only: every result is the same at any count. */
int ora_set_num_threads(int n) {
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
    return ora_num_threads();
}

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* sum_i a[i] * W[n][i] for an MXFP4 row: codes [K/2], scales [K/32]. */
static double dot_mxfp4(const uint8_t *codes, const uint8_t *scales, const double *a, int K,
                        const double *lut) {
    double acc = 0.0;
    for (int b = 0; b < K / 32; ++b) {
        double blk = 0.0;
        for (int i = 0; i < 32; ++i) {
            const int n = b * 32 + i;
            const uint8_t byte = codes[n / 2];
            blk += a[n] * lut[(n & 1) ? (byte >> 4) : (byte & 15)];
        }
        acc += blk * ora_e8m0_value(scales[b]);
    }
    return acc;
}

/* sum_i a[i] * W[n][i] for a Q2_K row of K/256 super-blocks. */
static double dot_q2k(const uint8_t *blocks, const double *a, int K) {
    float w[ORA_Q2K_BLOCK];
    double acc = 0.0;
    for (int b = 0; b < K / ORA_Q2K_BLOCK; ++b) {
        ora_q2k_dequantize(blocks + (int64_t)b * ORA_Q2K_BYTES, 1, ORA_Q2K_BLOCK, w);
        for (int i = 0; i < ORA_Q2K_BLOCK; ++i) acc += a[b * ORA_Q2K_BLOCK + i] * (double)w[i];
    }
    return acc;
}

static double dot_expert(const ora_layer *L, const uint8_t *codes, const uint8_t *scales,
                         int64_t row, const double *a, int K, const double *lut) {
    if (L->wfmt == ORA_W_Q2K)
        return dot_q2k(codes + row * (K / ORA_Q2K_BLOCK) * ORA_Q2K_BYTES, a, K);
    return dot_mxfp4(codes + row * (K / 2), scales + row * (K / 32), a, K, lut);
}

/* Quantise a vector along its length to MXFP8 and back (w4a8 activations). */
static void mxfp8_roundtrip(double *v, int K) {
    uint8_t *c = (uint8_t *)malloc((size_t)K), *s = (uint8_t *)malloc((size_t)K / 32);
    ora_mxfp8_quantize_f64(v, 1, K, c, s);
    ora_mxfp8_dequantize(c, s, 1, K, v);
    free(c);
    free(s);
}

/* The same with MXFP4 (w4a4 activations). */
static void mxfp4_roundtrip(double *v, int K) {
    uint8_t *c = (uint8_t *)malloc((size_t)K / 2), *s = (uint8_t *)malloc((size_t)K / 32);
    float *f = (float *)malloc(sizeof(float) * (size_t)K);
    ora_mxfp4_quantize_f64(v, 1, K, c, s);
    ora_mxfp4_dequantize(c, s, 1, K, f);  /* E2M1 x 2^e: exact in fp32 */
    for (int i = 0; i < K; ++i) v[i] = (double)f[i];
    free(c);
    free(s);
    free(f);
}

void ora_expert_ffn_token(const ora_layer *L, int e, const uint16_t *x_t, double *o) {
    const int d = L->d, F = L->F;
    double lut[16];
    for (int c = 0; c < 16; ++c) lut[c] = ora_e2m1_value((uint8_t)c);
    double *a = (double *)malloc(sizeof(double) * (size_t)d);
    double *h = (double *)malloc(sizeof(double) * (size_t)F);
    for (int i = 0; i < d; ++i) a[i] = ora_bf16_value(x_t[i]);
    if (L->act == ORA_A_MXFP8) mxfp8_roundtrip(a, d);
    if (L->act == ORA_A_MXFP4) mxfp4_roundtrip(a, d);

    const int64_t eF = (int64_t)e * F, ed = (int64_t)e * d;
    for (int n = 0; n < F; ++n) {
        const double g = dot_expert(L, L->w1, L->w1s, eF + n, a, d, lut);
        const double u = dot_expert(L, L->w3, L->w3s, eF + n, a, d, lut);
        h[n] = silu(g) * u;
    }
    if (L->act == ORA_A_MXFP8) mxfp8_roundtrip(h, F);
    else if (L->act == ORA_A_MXFP4) mxfp4_roundtrip(h, F);
    else
        for (int n = 0; n < F; ++n) h[n] = ora_bf16_value(ora_f64_to_bf16(h[n]));
    for (int i = 0; i < d; ++i) o[i] = dot_expert(L, L->w2, L->w2s, ed + i, h, F, lut);
    free(a);
    free(h);
}

void ora_shared_ffn_token(const ora_layer *L, const uint16_t *x_t, double *s) {
    const int d = L->d, Fs = L->Fs;
    double *h = (double *)malloc(sizeof(double) * (size_t)Fs);
    for (int n = 0; n < Fs; ++n) {
        double g = 0.0, u = 0.0;
        for (int i = 0; i < d; ++i) {
            const double xi = ora_bf16_value(x_t[i]);
            g += xi * ora_bf16_value(L->sw1[(int64_t)n * d + i]);
            u += xi * ora_bf16_value(L->sw3[(int64_t)n * d + i]);
        }
        h[n] = ora_bf16_value(ora_f64_to_bf16(silu(g) * u));
    }
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int n = 0; n < Fs; ++n) acc += h[n] * ora_bf16_value(L->sw2[(int64_t)i * Fs + n]);
        s[i] = acc;
    }
    free(h);
}

/* Expert outputs for permuted rows [row_begin, row_end): row r holds slot
 * perm[r] = t*k + j of expert e with offsets[e] <= r < offsets[e+1]. */
void ora_expert_ffn_rows(const ora_layer *L, const uint16_t *x, const int32_t *offsets,
                         const int32_t *perm, int64_t row_begin, int64_t row_end, float *out) {
    const int d = L->d;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = row_begin; r < row_end; ++r) {
        int e = 0;
        while (!(offsets[e] <= r && r < offsets[e + 1])) ++e;
        const int t = perm[r] / L->k;
        double *o = (double *)malloc(sizeof(double) * (size_t)d);
        ora_expert_ffn_token(L, e, x + (int64_t)t * d, o);
        for (int i = 0; i < d; ++i) out[(r - row_begin) * d + i] = (float)o[i];
        free(o);
    }
}

void ora_combine(const float *out_rows, const int32_t *inv_perm, const float *topk_w,
                 const float *shared, int T, int d, int k, float *y) {
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        for (int i = 0; i < d; ++i) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) {
                const int64_t s = (int64_t)t * k + j;
                acc += (double)topk_w[s] * (double)out_rows[(int64_t)inv_perm[s] * d + i];
            }
            if (shared) acc += (double)shared[(int64_t)t * d + i];
            y[(int64_t)t * d + i] = (float)acc;
        }
}

/* The whole layer for the chosen tokens (indices into x / token_ids): routing,
 * the k expert FFNs, the shared expert and the gate-weighted sum. Writes
 * idx/w [n][k] and y [n][d]. Returns the number of tokens whose hash routing
 * hit the draw cap (0 normally). */
int ora_layer_tokens(const ora_layer *L, const uint16_t *x, const int32_t *token_ids,
                     const int32_t *tokens, int n_tokens, int32_t *idx, float *w, float *y) {
    const int d = L->d, k = L->k, E = L->E;
    int failed = 0;
    for (int q = 0; q < n_tokens; ++q) {
        const int t = tokens[q];
        if (L->route == ORA_ROUTE_HASH) {
            failed += ora_hash_route(token_ids + t, 1, E, k, L->max_draws, idx + (int64_t)q * k,
                                     w + (int64_t)q * k);
        } else {
            float *logits = (float *)malloc(sizeof(float) * (size_t)E);
            ora_router_logits(x + (int64_t)t * d, L->wr, L->bias, 1, d, E, logits);
            ora_topk_softmax(logits, 1, E, k, idx + (int64_t)q * k, w + (int64_t)q * k);
            free(logits);
        }
    }
    const int64_t npairs = (int64_t)n_tokens * k;
    double *o = (double *)malloc(sizeof(double) * (size_t)(npairs + (L->Fs ? n_tokens : 0)) * d);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t p = 0; p < npairs + (L->Fs ? n_tokens : 0); ++p) {
        if (p < npairs) {
            const int q = (int)(p / k), e = idx[p];
            if (e >= 0) ora_expert_ffn_token(L, e, x + (int64_t)tokens[q] * d, o + p * d);
            else memset(o + p * d, 0, sizeof(double) * (size_t)d);
        } else {
            const int q = (int)(p - npairs);
            ora_shared_ffn_token(L, x + (int64_t)tokens[q] * d, o + p * d);
        }
    }
    for (int q = 0; q < n_tokens; ++q)
        for (int i = 0; i < d; ++i) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) acc += (double)w[(int64_t)q * k + j] * o[((int64_t)q * k + j) * d + i];
            if (L->Fs) acc += o[(npairs + q) * d + i];
            y[(int64_t)q * d + i] = (float)acc;
        }
    free(o);
    return failed;
}
