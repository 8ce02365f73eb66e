/*
 * Oracle routing: router logits, top-k softmax gates, hash routing.
 *
 * TEST INFRASTRUCTURE (see oracle.h).
 *
 * The router stays unquantised ("DS4", dibi8.com, "Key architectural
 * innovations" item 1; "DwarfStar", hysenlabs.com, "Model support and
 * quantisation"): logits are bf16 x times bf16 W_r with fp32 accumulation.
 * The model routes by hashing ("DeepSeek V4 Flash ... on a Mac", grapeot.me,
 * opening section); the pages do not give the hash, so the hash variant below
 * is the reading stated at ora_hash_route.
 *
 * Logits decide integers (which experts), so they are computed in fp32 in one
 * fixed order, the one the GPU kernel must reproduce bit for bit:
 *   K = d is cut into 32 contiguous chunks of d/32; chunk c's partial sum is a
 *   running fmaf from +0.0f over ascending i; the 32 partials are then summed
 *   as a balanced tree of adjacent pairs ((p0+p1)+(p2+p3))+...; the bias, when
 *   present, is added last.
 */
#include <math.h>
#include <string.h>

#include "oracle.h"

static float bf16f(uint16_t b) {
    const uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

void ora_router_logits(const uint16_t *x, const uint16_t *wr, const float *bias, int T, int d,
                       int E, float *logits) {
    const int chunk = d / 32;
#pragma omp parallel for collapse(2) schedule(static)
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            const uint16_t *xt = x + (int64_t)t * d, *we = wr + (int64_t)e * d;
            float p[32];
            for (int c = 0; c < 32; ++c) {
                float acc = 0.0f;
                for (int i = c * chunk; i < (c + 1) * chunk; ++i) acc = fmaf(bf16f(xt[i]), bf16f(we[i]), acc);
                p[c] = acc;
            }
            for (int w = 1; w < 32; w *= 2)
                for (int c = 0; c < 32; c += 2 * w) p[c] = p[c] + p[c + w];
            float l = p[0];
            if (bias) l = l + bias[e];
            logits[(int64_t)t * E + e] = l;
        }
}

/* Is expert a ranked before expert b? Larger logit first, NaN after every
 * number, equal logits (including +0 == -0) by the lower index. */
static int ranks_before(const float *l, int a, int b) {
    const int na = isnan(l[a]), nb = isnan(l[b]);
    if (na != nb) return nb;
    if (!na && l[a] != l[b]) return l[a] > l[b];
    return a < b;
}

/* Top-k by the order above, written in rank order; gates are the softmax of
 * the k selected logits (the same as a softmax over all E renormalised over
 * the selected k), computed in fp64. */
void ora_topk_softmax(const float *logits, int T, int E, int k, int32_t *idx, float *w) {
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        const float *l = logits + (int64_t)t * E;
        int32_t *it = idx + (int64_t)t * k;
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                int taken = 0;
                for (int q = 0; q < j; ++q) taken |= (it[q] == e);
                if (taken) continue;
                if (best < 0 || ranks_before(l, e, best)) best = e;
            }
            it[j] = best;
        }
        double den = 0.0, ex[1024];
        for (int j = 0; j < k; ++j) {
            ex[j] = exp((double)l[it[j]] - (double)l[it[0]]);
            den += ex[j];
        }
        for (int j = 0; j < k; ++j) w[(int64_t)t * k + j] = (float)(ex[j] / den);
    }
}

/* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014): the state advances by the odd constant
 * floor(2^64 / golden ratio) and each output is the state passed through a
 * xor-shift/multiply finaliser. */
uint64_t ora_splitmix64_next(uint64_t *state) {
    uint64_t z = (*state += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* Hash routing, reading: seed a SplitMix64 state with the token id
 * (zero-extended from 32 bits); draw outputs z_0, z_1, ...; expert = z mod E;
 * an expert already chosen for this token is skipped; stop at k accepted
 * experts, kept in acceptance order; every gate is 1/k. A token that needs
 * more than max_draws draws gets -1 in its unfilled slots and is counted in
 * the return value. */
int ora_hash_route(const int32_t *token_ids, int T, int E, int k, int max_draws, int32_t *idx,
                   float *w) {
    int failed = 0;
    for (int t = 0; t < T; ++t) {
        uint64_t st = (uint64_t)(uint32_t)token_ids[t];
        int32_t *it = idx + (int64_t)t * k;
        int n = 0, draws = 0;
        while (n < k && draws < max_draws) {
            const int e = (int)(ora_splitmix64_next(&st) % (uint64_t)E);
            ++draws;
            int dup = 0;
            for (int q = 0; q < n; ++q) dup |= (it[q] == e);
            if (!dup) it[n++] = e;
        }
        if (n < k) {
            ++failed;
            for (; n < k; ++n) it[n] = -1;
        }
        for (int j = 0; j < k; ++j) w[(int64_t)t * k + j] = 1.0f / (float)k;
    }
    return failed;
}
