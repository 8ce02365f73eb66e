/*
 * Oracle for the routed mixture-of-experts FFN layer over block-quantised
 * expert weights.
 *
 * TEST INFRASTRUCTURE. A plain, slow CPU restatement of what the layer
 * computes, used only by the test suite, the smoke check and the benchmark's
 * CPU-baseline leg. It shares no code with the CUDA library and the library
 * never calls it.
 *
 * Sources (DwarfStar 4 / DeepSeek V4 Flash pages):
 *  - "DeepSeek V4 Flash ... on a Mac" (grapeot.me), opening section: the model
 *    ships FP4+FP8 mixed weights and uses hash MoE routing;
 *  - "DS4 ..." (dibi8.com), "Key architectural innovations" item 1: the 2-bit
 *    build quantises only the routed experts (IQ2_XXS up/gate, Q2_K down) and
 *    keeps the shared experts, projections and router unquantised;
 *  - "DwarfStar" (hysenlabs.com), "Model support and quantisation": MXFP4 keeps
 *    the released routed-expert weights, and Blackwell batches expert work on
 *    native FP4 matrix instructions.
 * The pages give no formulas; each function states the definition it uses.
 * Floating point is fp64 except where a result decides an integer (router
 * logits -> top-k): those are fp32 in the fixed reduction order below.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- number formats (formats.c) ---------------------------------------- */
double ora_e2m1_value(uint8_t code);            /* OCP MX FP4 E2M1, low 4 bits */
double ora_e8m0_value(uint8_t e);               /* 2^(e-127); 0xFF -> NaN */
double ora_e4m3_value(uint8_t code);            /* OCP FP8 E4M3; S.1111.111 -> NaN */
uint8_t ora_e2m1_encode(double y);              /* RNE, saturating, sign kept */
uint8_t ora_e2m1_encode_nearest(double y);      /* same, by exhaustive search */
uint8_t ora_e4m3_encode(double y);              /* RNE, saturating to 448, sign kept */
uint8_t ora_e4m3_encode_nearest(double y);      /* same, by exhaustive search */
int ora_floor_log2(double a);                   /* a > 0, from the binary exponent */

uint16_t ora_f32_to_f16(float v);               /* IEEE binary16, RNE */
double ora_f16_value(uint16_t h);
uint16_t ora_f64_to_bf16(double v);             /* bfloat16, RNE */
double ora_bf16_value(uint16_t b);

/* MXFP4: 32-element blocks along K. codes [rows][K/2] (element 2i in the low
 * nibble), scales [rows][K/32] E8M0. */
void ora_mxfp4_quantize(const float *w, int64_t rows, int64_t K, uint8_t *codes, uint8_t *scales);
void ora_mxfp4_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t K,
                          float *out);
/* The same rule on fp64 values (MXFP4 activations, "w4a4"). */
void ora_mxfp4_quantize_f64(const double *v, int64_t rows, int64_t K, uint8_t *codes, uint8_t *scales);
/* MXFP8 (E4M3 elements): codes [rows][K], scales [rows][K/32]. */
void ora_mxfp8_quantize_f64(const double *v, int64_t rows, int64_t K, uint8_t *codes,
                            uint8_t *scales);
void ora_mxfp8_quantize_bf16(const uint16_t *x, int64_t rows, int64_t K, uint8_t *codes,
                             uint8_t *scales);
void ora_mxfp8_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t K,
                          double *out);
/* Q2_K-style: 256-weight super-blocks of 84 bytes along K. */
#define ORA_Q2K_BLOCK 256
#define ORA_Q2K_BYTES 84
void ora_q2k_quantize(const float *w, int64_t rows, int64_t K, uint8_t *blocks);
void ora_q2k_dequantize(const uint8_t *blocks, int64_t rows, int64_t K, float *out);

/* ---- routing (route.c) ------------------------------------------------- */
void ora_router_logits(const uint16_t *x, const uint16_t *wr, const float *bias, int T, int d,
                       int E, float *logits);
void ora_topk_softmax(const float *logits, int T, int E, int k, int32_t *idx, float *w);
uint64_t ora_splitmix64_next(uint64_t *state);
int ora_hash_route(const int32_t *token_ids, int T, int E, int k, int max_draws, int32_t *idx,
                   float *w);

/* ---- permute (permute.c) ----------------------------------------------- */
int ora_permute(const int32_t *idx, int T, int k, int E, int32_t *counts, int32_t *offsets,
                int32_t *perm, int32_t *inv_perm);

/* ---- expert FFN, combine, layer (ffn.c) -------------------------------- */
enum { ORA_W_MXFP4 = 1, ORA_W_Q2K = 2 };
enum { ORA_A_BF16 = 0, ORA_A_MXFP8 = 1, ORA_A_MXFP4 = 2 };
enum { ORA_ROUTE_SOFTMAX = 0, ORA_ROUTE_HASH = 1 };

typedef struct {
    int32_t T, d, F, E, k;
    int32_t wfmt;   /* ORA_W_* */
    int32_t act;    /* ORA_A_* */
    int32_t route;  /* ORA_ROUTE_* */
    int32_t Fs;     /* shared expert d_ff, 0 = none */
    int32_t max_draws;
    /* routed experts, canonical layout. MXFP4: codes + scales. Q2_K: blocks in
     * w1/w3/w2, scale pointers unused. W1, W3: [E][F][d]; W2: [E][d][F]. */
    const uint8_t *w1, *w1s, *w3, *w3s, *w2, *w2s;
    /* shared expert, bf16 bits: [Fs][d], [Fs][d], [d][Fs] */
    const uint16_t *sw1, *sw3, *sw2;
    const uint16_t *wr;   /* router [E][d] bf16 bits */
    const float *bias;    /* [E] or NULL */
} ora_layer;

void ora_expert_ffn_token(const ora_layer *L, int e, const uint16_t *x_t, double *o);
void ora_shared_ffn_token(const ora_layer *L, const uint16_t *x_t, double *s);
void ora_expert_ffn_rows(const ora_layer *L, const uint16_t *x, const int32_t *offsets,
                         const int32_t *perm, int64_t row_begin, int64_t row_end, float *out);
void ora_combine(const float *out_rows, const int32_t *inv_perm, const float *topk_w,
                 const float *shared, int T, int d, int k, float *y);
int ora_layer_tokens(const ora_layer *L, const uint16_t *x, const int32_t *token_ids,
                     const int32_t *tokens, int n_tokens, int32_t *idx, float *w, float *y);

int ora_num_threads(void);
int ora_set_num_threads(int n);   /* threading only; returns the count in effect */

#ifdef __cplusplus
}
#endif
#endif
