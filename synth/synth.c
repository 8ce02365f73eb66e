/*
 * Seeded synthetic inputs for the routed expert FFN layer.
 *
 * Test and benchmark infrastructure, shared by the oracle side and the CUDA
 * side. This file only draws random numbers and shapes them into the
 * workloads' distributions (normal, uniform integers, permutations). It holds
 * none of the layer's arithmetic: no quantisation, routing, permutation or FFN
 * math lives here.
 *
 * Generator: Philox4x32-10, the counter-based generator of Salmon, Moraes,
 * Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3" (SC'11).
 * Every value is a pure function of (seed, tensor, sub, index), so experts and
 * token batches can be generated independently and in parallel.
 *
 *   key     = (low 32 bits of seed, tensor id)
 *   counter = (block index low, block index high, sub, kind)
 *
 * kind 0 = normals (Box-Muller, one block -> two normals),
 * kind 1 = uniforms (one block -> two 53-bit uniforms).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static inline void philox_round(uint32_t x[4], uint32_t k0, uint32_t k1) {
    const uint64_t p0 = (uint64_t)0xD2511F53u * x[0];
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * x[2];
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    const uint32_t y0 = hi1 ^ x[1] ^ k0;
    const uint32_t y2 = hi0 ^ x[3] ^ k1;
    x[0] = y0;
    x[1] = lo1;
    x[2] = y2;
    x[3] = lo0;
}

void synth_philox4x32_10(const uint32_t ctr[4], uint32_t k0, uint32_t k1, uint32_t out[4]) {
    uint32_t x[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
    for (int r = 0; r < 10; ++r) {
        if (r) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        philox_round(x, k0, k1);
    }
    memcpy(out, x, sizeof x);
}

static inline void block(uint64_t seed, uint32_t tensor, uint32_t sub, uint32_t kind,
                         uint64_t b, uint32_t out[4]) {
    const uint32_t ctr[4] = {(uint32_t)b, (uint32_t)(b >> 32), sub, kind};
    synth_philox4x32_10(ctr, (uint32_t)seed, tensor ^ (uint32_t)(seed >> 32), out);
}

/* 53-bit uniform strictly inside (0, 1). */
static inline double u53(uint32_t hi, uint32_t lo) {
    const uint64_t v = (((uint64_t)hi << 32) | lo) >> 11;
    return ((double)v + 0.5) * 0x1.0p-53;
}

static inline double normal_at(uint64_t seed, uint32_t tensor, uint32_t sub, uint64_t j) {
    uint32_t r[4];
    block(seed, tensor, sub, 0u, j >> 1, r);
    const double u1 = u53(r[0], r[1]);
    const double u2 = u53(r[2], r[3]);
    const double rad = sqrt(-2.0 * log(u1));
    const double ang = 6.283185307179586476925286766559 * u2;
    return (j & 1) ? rad * sin(ang) : rad * cos(ang);
}

/* Both normals of Box-Muller pair b (normals 2b and 2b+1). */
static inline void normal_pair(uint64_t seed, uint32_t tensor, uint32_t sub, uint64_t b, double z[2]) {
    uint32_t r[4];
    block(seed, tensor, sub, 0u, b, r);
    const double u1 = u53(r[0], r[1]);
    const double u2 = u53(r[2], r[3]);
    const double rad = sqrt(-2.0 * log(u1));
    const double ang = 6.283185307179586476925286766559 * u2;
    z[0] = rad * cos(ang);
    z[1] = rad * sin(ang);
}

/* out[i] = (float)(mean + std * z_{first+i}) */
void synth_normal_f32(uint64_t seed, uint32_t tensor, uint32_t sub, uint64_t first, int64_t n,
                      double mean, double std, float *out) {
    if (n <= 0) return;
    const uint64_t b0 = first >> 1, b1 = (first + (uint64_t)n + 1) >> 1;
#pragma omp parallel for schedule(static)
    for (int64_t b = (int64_t)b0; b < (int64_t)b1; ++b) {
        double z[2];
        normal_pair(seed, tensor, sub, (uint64_t)b, z);
        for (int h = 0; h < 2; ++h) {
            const int64_t i = 2 * b + h - (int64_t)first;
            if (i >= 0 && i < n) out[i] = (float)(mean + std * z[h]);
        }
    }
}

/* bfloat16 bit pattern of the float value above, round-to-nearest-even. */
static inline uint16_t to_bf16_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

void synth_normal_bf16(uint64_t seed, uint32_t tensor, uint32_t sub, uint64_t first, int64_t n,
                       double mean, double std, uint16_t *out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = to_bf16_bits((float)(mean + std * normal_at(seed, tensor, sub, first + (uint64_t)i)));
}

static inline double uniform_at(uint64_t seed, uint32_t tensor, uint32_t sub, uint64_t j) {
    uint32_t r[4];
    block(seed, tensor, sub, 1u, j >> 1, r);
    return (j & 1) ? u53(r[2], r[3]) : u53(r[0], r[1]);
}

void synth_uniform_f64(uint64_t seed, uint32_t tensor, uint32_t sub, uint64_t first, int64_t n,
                       double *out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = uniform_at(seed, tensor, sub, first + (uint64_t)i);
}

/* Integers uniform in [lo, hi). */
void synth_uniform_int(uint64_t seed, uint32_t tensor, uint32_t sub, uint64_t first, int64_t n,
                       int64_t lo, int64_t hi, int32_t *out) {
    const double span = (double)(hi - lo);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        int64_t v = lo + (int64_t)floor(uniform_at(seed, tensor, sub, first + (uint64_t)i) * span);
        if (v >= hi) v = hi - 1;
        out[i] = (int32_t)v;
    }
}

/* A uniformly random permutation of 0..n-1 (Fisher-Yates, descending). */
void synth_permutation(uint64_t seed, uint32_t tensor, uint32_t sub, int32_t n, int32_t *out) {
    for (int32_t i = 0; i < n; ++i) out[i] = i;
    for (int32_t i = n - 1; i > 0; --i) {
        int32_t j = (int32_t)floor(uniform_at(seed, tensor, sub, (uint64_t)i) * (double)(i + 1));
        if (j > i) j = i;
        const int32_t t = out[i];
        out[i] = out[j];
        out[j] = t;
    }
}

int synth_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
