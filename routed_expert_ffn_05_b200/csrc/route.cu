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
// balanced tree of adjacent pairs; the bias is added last. Batches of 32
// tokens or more take the tensor-core router (router_tc.cu), which reaches
// the same expert choice; smaller batches the per-token kernel below.
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

// One warp per token: k rounds of a warp arg-max over the unchosen experts,
// then the softmax of the k chosen logits.
__global__ void __launch_bounds__(256) topk_softmax_kernel(const float *__restrict__ logits, int T,
                                                           int E, int k, int32_t *__restrict__ idx,
                                                           float *__restrict__ w) {
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (t >= T) return;
    const float *l = logits + (int64_t)t * E;
    const int my_e = topk_row(l, E, k, lane);
    const float my_l = lane < k ? l[my_e] : 0.f;
    const float l0 = __shfl_sync(0xffffffffu, my_l, 0);
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
__global__ void hash_route_kernel(const int32_t *__restrict__ token_ids, int T, int E, int k, int max_draws,
                                  int32_t *__restrict__ idx, float *__restrict__ w, int *err) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    uint64_t st = (uint64_t)(uint32_t)token_ids[t];
    int32_t chosen[32];
    int n = 0;
    for (int draws = 0; n < k && draws < max_draws; ++draws) {
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

cudaError_t launch_hash_route(const moe_dims &d, const int32_t *token_ids, int max_draws, int32_t *idx, float *w,
                              cudaStream_t s) {
    if (d.T == 0) return cudaSuccess;
    hash_route_kernel<<<ceil_div(d.T, 128), 128, 0, s>>>(token_ids, d.T, d.E, d.k, max_draws, idx, w,
                                                          device_error_word());
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_route(const moe_dims &d, const uint16_t *x, const moe_weights &wt,
                         const int32_t *token_ids, int32_t *idx, float *w, float *logits, float *rnorm,
                         cudaStream_t s) {
    if (d.T == 0) return cudaSuccess;
    if (d.route == MOE_ROUTE_HASH) return launch_hash_route(d, token_ids, kHashMaxDraws, idx, w, s);
    if (router_tc_applies(d)) return launch_route_tc(d, x, wt, idx, w, logits, rnorm, s);
    const int ey = ceil_div(d.E, 8);
    router_logits_kernel<<<dim3(d.T, ey), 256, d.d_model * 2, s>>>(x, wt.w_router, wt.router_bias, d.T,
                                                                      d.d_model, d.E, logits);
    topk_softmax_kernel<<<ceil_div(d.T, 8), 256, 0, s>>>(logits, d.T, d.E, d.k, idx, w);
    count_launches(2);
    return cudaGetLastError();
}

}  // namespace moe
