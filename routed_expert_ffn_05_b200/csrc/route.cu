// Routing: router logits in a fixed fp32 order, top-k with softmax gates, and
// hash routing.
//
// The router is unquantised bf16 ("DS4", dibi8.com, "Key architectural
// innovations" item 1). The model routes by hashing ("DeepSeek V4 Flash ... on
// a Mac", grapeot.me, opening section); the hash is SplitMix64 (Steele, Lea and
// Flood, OOPSLA 2014) seeded with the token id.
//
// Logit order (it decides integers, so it is fixed): K = d is cut into 32
// contiguous chunks; lane c of a warp runs the fma chain of chunk c from +0.0,
// then a butterfly over lanes with offsets 1, 2, 4, 8, 16 sums the chunks as a
// balanced tree of adjacent pairs; the bias is added last.
#include "common.cuh"
#include "kernels.h"

namespace moe {

// Decode-sized router: one warp per (token, expert), the token's x row staged
// once per block in shared memory.
__global__ void __launch_bounds__(256) router_logits_kernel(const uint16_t *__restrict__ x,
                                                            const uint16_t *__restrict__ wr,
                                                            const float *__restrict__ bias, int T,
                                                            int d, int E, float *__restrict__ logits) {
    extern __shared__ uint16_t xs_smem[];
    const int t = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint4 *xr = reinterpret_cast<const uint4 *>(x + (int64_t)t * d);
    uint4 *xs4 = reinterpret_cast<uint4 *>(xs_smem);
    for (int i = threadIdx.x; i < d / 8; i += blockDim.x) xs4[i] = xr[i];
    __syncthreads();
    const int chunk = d / 32;
    for (int e = blockIdx.y * 8 + warp; e < E; e += gridDim.y * 8) {
        const uint4 *w4 = reinterpret_cast<const uint4 *>(wr + (int64_t)e * d + lane * chunk);
        const uint4 *x4 = reinterpret_cast<const uint4 *>(xs_smem + lane * chunk);
        float acc = 0.0f;
        for (int v = 0; v < chunk / 8; ++v) {
            const uint4 wv = __ldg(w4 + v), xv = x4[v];
            const uint32_t wa[4] = {wv.x, wv.y, wv.z, wv.w}, xa[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc = __fmaf_rn(__uint_as_float(xa[q] << 16), __uint_as_float(wa[q] << 16), acc);
                acc = __fmaf_rn(__uint_as_float(xa[q] & 0xFFFF0000u), __uint_as_float(wa[q] & 0xFFFF0000u), acc);
            }
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
        if (lane == 0) logits[(int64_t)t * E + e] = bias ? __fadd_rn(acc, bias[e]) : acc;
    }
}

// Batch router: a CTA covers 32 tokens x 16 experts; warp w takes 8 tokens x 8
// experts and lane c the chunk c of every one of its 64 dot products, so each
// (token, expert) still runs the fixed order above (fma chain per chunk, then
// the butterfly). Operands are staged per 8-element step of all 32 chunks, as
// fp32, in [row][half][chunk][4] order: lane c reads 16 contiguous bytes, so a
// warp's loads hit distinct banks. Requires d % 256 == 0.
constexpr int kRtT = 32, kRtE = 16;
constexpr int kRtXs = kRtT * 2 * 32 * 4, kRtWs = kRtE * 2 * 32 * 4;  // floats per buffer
constexpr int kRtSmem = 2 * (kRtXs + kRtWs) * 4;

__global__ void __launch_bounds__(256, 1) router_tiled_kernel(const uint16_t *__restrict__ x,
                                                              const uint16_t *__restrict__ wr,
                                                              const float *__restrict__ bias, int T, int d,
                                                              int E, float *__restrict__ logits) {
    extern __shared__ float4 rt_smem[];
    float *xs = reinterpret_cast<float *>(rt_smem), *ws = xs + 2 * kRtXs;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t_base = blockIdx.y * kRtT, e_base = blockIdx.x * kRtE;
    const int chunk = d / 32, steps = chunk / 8;
    // staging: 32 x-rows and 16 w-rows, 32 chunks each, 8 bf16 per (row, chunk)
    auto load = [&](int st, uint4 (&v)[6]) {
#pragma unroll
        for (int q = 0; q < 6; ++q) {
            const int i = threadIdx.x + 256 * q;  // (row, chunk): rows 0..31 x, 32..47 w
            const int row = i >> 5, c = i & 31;
            const bool isx = row < kRtT;
            const int g = isx ? t_base + row : e_base + row - kRtT;
            const bool in = g < (isx ? T : E);
            const uint16_t *src = (isx ? x : wr) + (int64_t)g * d + c * chunk + 8 * st;
            v[q] = in ? __ldg(reinterpret_cast<const uint4 *>(src)) : make_uint4(0, 0, 0, 0);
        }
    };
    auto store = [&](int buf, const uint4 (&v)[6]) {
#pragma unroll
        for (int q = 0; q < 6; ++q) {
            const int i = threadIdx.x + 256 * q;
            const int row = i >> 5, c = i & 31;
            float *dst = row < kRtT ? xs + buf * kRtXs + (row * 2) * 128 + c * 4
                                    : ws + buf * kRtWs + ((row - kRtT) * 2) * 128 + c * 4;
            const uint32_t a[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
            reinterpret_cast<float4 *>(dst)[0] = make_float4(__uint_as_float(a[0] << 16), __uint_as_float(a[0] & 0xFFFF0000u),
                                                             __uint_as_float(a[1] << 16), __uint_as_float(a[1] & 0xFFFF0000u));
            reinterpret_cast<float4 *>(dst + 128)[0] = make_float4(__uint_as_float(a[2] << 16), __uint_as_float(a[2] & 0xFFFF0000u),
                                                                   __uint_as_float(a[3] << 16), __uint_as_float(a[3] & 0xFFFF0000u));
        }
    };
    const int tw = (warp >> 1) * 8, ew = (warp & 1) * 8;  // this warp's 8 tokens, 8 experts
    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.0f;
    uint4 v[6];
    load(0, v);
    store(0, v);
    __syncthreads();
    for (int st = 0; st < steps; ++st) {
        const int buf = st & 1;
        if (st + 1 < steps) load(st + 1, v);
        const float *xb = xs + buf * kRtXs, *wb = ws + buf * kRtWs;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float4 xv[8], wv[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) xv[a] = reinterpret_cast<const float4 *>(xb + ((tw + a) * 2 + h) * 128)[lane];
#pragma unroll
            for (int b = 0; b < 8; ++b) wv[b] = reinterpret_cast<const float4 *>(wb + ((ew + b) * 2 + h) * 128)[lane];
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) {
                    acc[a][b] = __fmaf_rn(xv[a].x, wv[b].x, acc[a][b]);
                    acc[a][b] = __fmaf_rn(xv[a].y, wv[b].y, acc[a][b]);
                    acc[a][b] = __fmaf_rn(xv[a].z, wv[b].z, acc[a][b]);
                    acc[a][b] = __fmaf_rn(xv[a].w, wv[b].w, acc[a][b]);
                }
        }
        if (st + 1 < steps) store(buf ^ 1, v);
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            float p = acc[a][b];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) p = __fadd_rn(p, __shfl_xor_sync(0xffffffffu, p, o));
            acc[a][b] = p;
        }
    // every lane holds every sum now; lane (8a + b) % 32 writes (tw + a, ew + b)
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const int t = t_base + tw + a, e = e_base + ew + b;
            if (lane == ((8 * a + b) & 31) && t < T && e < E)
                logits[(int64_t)t * E + e] = bias ? __fadd_rn(acc[a][b], bias[e]) : acc[a][b];
        }
}

// a ranks before b: larger logit first, NaN after every number, ties (and
// +0 == -0) by the lower index.
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
    const bool na = isnan(va), nb = isnan(vb);
    if (na != nb) return nb;
    if (!na && va != vb) return va > vb;
    return ia < ib;
}

// One warp per token: k rounds of a warp arg-max over the unchosen experts,
// then the softmax of the k chosen logits.
__global__ void __launch_bounds__(256) topk_softmax_kernel(const float *__restrict__ logits, int T,
                                                           int E, int k, int32_t *__restrict__ idx,
                                                           float *__restrict__ w) {
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (t >= T) return;
    const float *l = logits + (int64_t)t * E;
    uint32_t taken = 0;  // bit i: expert lane + 32 i chosen (E <= 1024)
    float my_l = 0.0f;
    int my_e = -1;
    float l0 = 0.0f;
    for (int j = 0; j < k; ++j) {
        float bv = 0.0f;
        int bi = -1;
        for (int i = 0, e = lane; e < E; ++i, e += 32) {
            if (taken >> i & 1u) continue;
            const float v = l[e];
            if (bi < 0 || ranks_before(v, e, bv, bi)) { bv = v; bi = e; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (oi >= 0 && (bi < 0 || ranks_before(ov, oi, bv, bi))) { bv = ov; bi = oi; }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (j == 0) l0 = bv;
        if (lane == j) { my_l = bv; my_e = bi; }
    }
    const float ex = lane < k ? expf(my_l - l0) : 0.0f;
    const float den = warp_sum(ex);
    if (lane < k) {
        idx[(int64_t)t * k + lane] = my_e;
        w[(int64_t)t * k + lane] = ex / den;
    }
}

__device__ __forceinline__ uint64_t splitmix64_next(uint64_t &s) {
    uint64_t z = (s += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// One thread per token: draw until k distinct experts are accepted; the
// draw cap turns a pathological id into a device error, never a hang.
__global__ void hash_route_kernel(const int32_t *__restrict__ token_ids, int T, int E, int k,
                                  int32_t *__restrict__ idx, float *__restrict__ w, int *err) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    uint64_t st = (uint64_t)(uint32_t)token_ids[t];
    int32_t chosen[32];
    int n = 0;
    for (int draws = 0; n < k && draws < kHashMaxDraws; ++draws) {
        const int e = (int)(splitmix64_next(st) % (uint64_t)E);
        bool dup = false;
        for (int q = 0; q < n; ++q) dup |= (chosen[q] == e);
        if (!dup) chosen[n++] = e;
    }
    if (n < k) set_device_error(err, MOE_DEVERR_HASH_CAP);
    const float g = 1.0f / (float)k;
    for (int j = 0; j < k; ++j) {
        idx[(int64_t)t * k + j] = j < n ? chosen[j] : -1;
        w[(int64_t)t * k + j] = g;
    }
}

cudaError_t launch_route(const moe_dims &d, const uint16_t *x, const moe_weights &wt,
                         const int32_t *token_ids, int32_t *idx, float *w, float *logits,
                         cudaStream_t s) {
    if (d.T == 0) return cudaSuccess;
    if (d.route == MOE_ROUTE_HASH) {
        hash_route_kernel<<<ceil_div(d.T, 128), 128, 0, s>>>(token_ids, d.T, d.E, d.k, idx, w,
                                                              device_error_word());
        count_launches(1);
        return cudaGetLastError();
    }
    if (d.T >= kRtT && d.d_model % 256 == 0) {
        static bool attr_set[64] = {false};
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev >= 0 && dev < 64 && !attr_set[dev]) {
            cudaError_t e = cudaFuncSetAttribute(router_tiled_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRtSmem);
            if (e != cudaSuccess) return e;
            attr_set[dev] = true;
        }
        router_tiled_kernel<<<dim3(ceil_div(d.E, kRtE), ceil_div(d.T, kRtT)), 256, kRtSmem, s>>>(
            x, wt.w_router, wt.router_bias, d.T, d.d_model, d.E, logits);
    } else {
        const int ey = ceil_div(d.E, 8);
        router_logits_kernel<<<dim3(d.T, ey), 256, d.d_model * 2, s>>>(x, wt.w_router, wt.router_bias, d.T,
                                                                          d.d_model, d.E, logits);
    }
    topk_softmax_kernel<<<ceil_div(d.T, 8), 256, 0, s>>>(logits, d.T, d.E, d.k, idx, w);
    count_launches(2);
    return cudaGetLastError();
}

}  // namespace moe
