// Shared device helpers of the routed MoE FFN library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// Kernels that can detect bad input get the device address of the per-device
// error word (first error wins); moe_get_device_error reads and clears it.
__device__ __forceinline__ void set_device_error(int *err, int code) { atomicCAS(err, 0, code); }

__host__ __device__ __forceinline__ int64_t align_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }
__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// fp32 -> bf16 bits, round to nearest even (inputs are finite here).
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)((u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u));
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

// E8M0 scale byte -> fp32 2^(e-127); 0xFF -> NaN. 2^-127 is an fp32 subnormal.
__device__ __forceinline__ float e8m0_to_f32(uint32_t e) {
    if (e == 0xFFu) return __uint_as_float(0x7FC00000u);
    if (e == 0u) return __uint_as_float(0x00400000u);
    return __uint_as_float(e << 23);
}

// floor(log2(a)) for a finite a > 0, from the binary exponent (subnormals too).
__device__ __forceinline__ int floor_log2_f32(float a) {
    const uint32_t u = __float_as_uint(a);
    const int e = (int)((u >> 23) & 0xFFu);
    if (e != 0) return e - 127;
    return (31 - __clz((int)(u & 0x7FFFFFu))) - 149;
}

// E2M1 magnitude codes 0..7 are 0, .5, 1, 1.5, 2, 3, 4, 6; bit 3 is the sign.
__device__ __forceinline__ float e2m1_to_f32(uint32_t c) {
    const uint32_t e = (c >> 1) & 3u, m = c & 1u;
    float mag = (e == 0) ? 0.5f * (float)m : __uint_as_float((e + 126u) << 23 | m << 22);
    return (c & 8u) ? -mag : mag;
}

// Two E2M1 codes (one byte, element 2i in the low nibble) -> two fp16 in one
// register, low half = low nibble (hardware conversion, exact).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
    uint32_t out;
    asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(out) : "r"(byte));
    return out;
}

// Slot range of expert e in the permuted order: binary search over offsets[E+1].
__device__ __forceinline__ int expert_of_row(const int32_t *offsets, int E, int row) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offsets[mid] <= row) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Routing order of (logit v, expert e): larger logit first, NaN after every
// number, ties (and +0 == -0) by the lower expert index. rank_word is the
// float made monotone as an unsigned word (-0 as +0, NaN as 0; every number
// maps above 0), so the order is: larger word first, then lower index.
__device__ __forceinline__ uint32_t rank_word(float v) {
    uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return isnan(v) ? 0u : u;
}

// Warp-wide top-k of one row of E <= 32 NC logits: lane holds cv[i] = logit
// of expert lane + 32 i. Pick j is the first unchosen expert in routing
// order, found in two 32-bit warp reductions: the largest rank_word, then the
// lowest unchosen expert index holding it. Lane j receives pick j. NC is a
// compile-time bound so the loops stay short (the kernels that use this run
// once per layer call, from a cold instruction cache).
template <int NC>
__device__ __forceinline__ int topk_warp(const float (&cv)[NC], int E, int k, int lane) {
    uint32_t u[NC], live = 0;  // live: bit i set while expert lane + 32 i is unchosen
#pragma unroll
    for (int i = 0; i < NC; ++i) {
        const bool in = lane + 32 * i < E;
        u[i] = in ? rank_word(cv[i]) : 0u;
        live |= in ? 1u << i : 0u;
    }
    int my_e = -1;
    for (int j = 0; j < k; ++j) {
        uint32_t best = 0;  // chosen and absent slots hold 0, at or below every live word
#pragma unroll
        for (int i = 0; i < NC; ++i) best = max(best, u[i]);
        const uint32_t m = __reduce_max_sync(0xffffffffu, best);
        uint32_t cand = 0xffffffffu;  // lowest live expert of this lane holding m
#pragma unroll
        for (int i = NC - 1; i >= 0; --i) cand = (u[i] == m && (live >> i & 1u)) ? (uint32_t)(lane + 32 * i) : cand;
        const int e = (int)__reduce_min_sync(0xffffffffu, cand);
        if ((e & 31) == lane) live &= ~(1u << (e >> 5));
#pragma unroll
        for (int i = 0; i < NC; ++i) u[i] = lane + 32 * i == e ? 0u : u[i];
        my_e = lane == j ? e : my_e;
    }
    return my_e;
}

// Top-k of the row l[0 .. E) (E <= 1024) by one warp; lane j gets pick j.
__device__ __forceinline__ int topk_row(const float *l, int E, int k, int lane) {
    if (E <= 256) {
        float cv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) cv[i] = lane + 32 * i < E ? l[lane + 32 * i] : 0.f;
        return topk_warp<8>(cv, E, k, lane);
    }
    float cv[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) cv[i] = lane + 32 * i < E ? l[lane + 32 * i] : 0.f;
    return topk_warp<32>(cv, E, k, lane);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// SiLU with the fast exponential and division intrinsics (relative error of a
// few ulp of fp32; h is rounded to bf16 or an 8-bit code right after). For
// g < -88 the exponential overflows to +Inf and the quotient is 0, the limit.
__device__ __forceinline__ float silu_f32(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

}  // namespace moe
