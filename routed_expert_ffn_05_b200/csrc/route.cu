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
__device__ __forceinline__ uint32_t smem_u32_rt(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
}  // namespace moe

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

// Batch router: a CTA covers 32 tokens x 32 experts; warp w takes 8 tokens x
// 16 experts and lane c the chunk c of each of its 128 dot products, so every
// (token, expert) still runs the fixed order above (fma chain per chunk, then
// the butterfly). Operands are copied as bf16 with cp.async, 8 elements of
// every chunk per step, in [row][chunk][8] order (lane c reads 8 contiguous
// bytes at a 16-byte stride), three steps in flight; values widen to fp32 on
// read. Requires d % 256 == 0.
constexpr int kRtT = 32, kRtE = 32, kRtStages = 3;
constexpr int kRtRowBytes = 32 * 16;                          // one row: 32 chunks x 8 bf16
constexpr int kRtStageBytes = (kRtT + kRtE) * kRtRowBytes;    // 32 KB
constexpr int kRtSmem = kRtStages * kRtStageBytes;

__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool in) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32_rt(dst)), "l"(src), "r"(in ? 16 : 0)
                 : "memory");
}

__global__ void __launch_bounds__(256, 1) router_tiled_kernel(const uint16_t *__restrict__ x,
                                                              const uint16_t *__restrict__ wr,
                                                              const float *__restrict__ bias, int T, int d,
                                                              int E, float *__restrict__ logits) {
    extern __shared__ uint4 rt_smem[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(rt_smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t_base = blockIdx.y * kRtT, e_base = blockIdx.x * kRtE;
    const int chunk = d / 32, steps = chunk / 8;
    // step st: rows 0..31 x, 32..63 w; 8 bf16 of every chunk; zero-filled past T / E
    auto issue = [&](int st) {
        uint8_t *dst0 = sm + (st % kRtStages) * kRtStageBytes;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int i = threadIdx.x + 256 * q;
            const int row = i >> 5, c = i & 31;
            const bool isx = row < kRtT;
            const int g = isx ? t_base + row : e_base + row - kRtT;
            const bool in = g < (isx ? T : E);
            const uint16_t *src = (isx ? x : wr) + (int64_t)(in ? g : 0) * d + c * chunk + 8 * st;
            cp_async16(dst0 + row * kRtRowBytes + c * 16, src, in);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    const int tw = (warp >> 1) * 8, ew = kRtT + (warp & 1) * 16;  // this warp's rows (x, w)
    float acc[8][16];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 16; ++b) acc[a][b] = 0.0f;
    for (int st = 0; st < kRtStages - 1; ++st) {
        if (st < steps) issue(st);
        else asm volatile("cp.async.commit_group;" ::: "memory");
    }
    for (int st = 0; st < steps; ++st) {
        asm volatile("cp.async.wait_group %0;" ::"n"(kRtStages - 2) : "memory");
        __syncthreads();
        if (st + kRtStages - 1 < steps) issue(st + kRtStages - 1);
        else asm volatile("cp.async.commit_group;" ::: "memory");
        const uint8_t *b0 = sm + (st % kRtStages) * kRtStageBytes + lane * 16;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint2 xp[8], wp[16];
#pragma unroll
            for (int a = 0; a < 8; ++a) xp[a] = *reinterpret_cast<const uint2 *>(b0 + (tw + a) * kRtRowBytes + 8 * h);
#pragma unroll
            for (int b = 0; b < 16; ++b) wp[b] = *reinterpret_cast<const uint2 *>(b0 + (ew + b) * kRtRowBytes + 8 * h);
#pragma unroll
            for (int j = 0; j < 4; ++j) {  // element 8 st + 4 h + j of every chunk, ascending
                float xf[8];
#pragma unroll
                for (int a = 0; a < 8; ++a) {
                    const uint32_t v = j < 2 ? xp[a].x : xp[a].y;
                    xf[a] = __uint_as_float((j & 1) ? (v & 0xFFFF0000u) : (v << 16));
                }
#pragma unroll
                for (int b = 0; b < 16; ++b) {
                    const uint32_t v = j < 2 ? wp[b].x : wp[b].y;
                    const float wf = __uint_as_float((j & 1) ? (v & 0xFFFF0000u) : (v << 16));
#pragma unroll
                    for (int a = 0; a < 8; ++a) acc[a][b] = __fmaf_rn(xf[a], wf, acc[a][b]);
                }
            }
        }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 16; ++b) {
            float p = acc[a][b];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) p = __fadd_rn(p, __shfl_xor_sync(0xffffffffu, p, o));
            acc[a][b] = p;
        }
    // every lane holds every sum now; lane (16a + b) % 32 writes (token tw + a, expert b)
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 16; ++b) {
            const int t = t_base + tw + a, e = e_base + (warp & 1) * 16 + b;
            if (lane == ((16 * a + b) & 31) && t < T && e < E)
                logits[(int64_t)t * E + e] = bias ? __fadd_rn(acc[a][b], bias[e]) : acc[a][b];
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
