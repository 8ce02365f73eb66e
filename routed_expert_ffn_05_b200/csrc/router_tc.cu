// Batch router (T >= 32 tokens, softmax top-k) on the tensor cores, with the
// expert choice still exact.
//
// The router is unquantised bf16 ("DS4", dibi8.com, "Key architectural
// innovations" item 1). Its logits decide integers, so the expert choice must
// be that of the canonical fp32 logits: 32 contiguous chunks of d/32, each a
// running fma from +0 in element order, a balanced tree of adjacent pairs
// (a warp butterfly with offsets 1, 2, 4, 8, 16), then the bias. Computing
// all T x E of them in that order ties the router to the CUDA cores. Instead:
//  1. router_approx_kernel: one bf16 GEMM on tcgen05 (kind::f16, fp32
//     accumulate in tensor memory) gives approximate logits a[t][e] for every
//     pair; extra CTAs compute the router rows' 2-norms |W_r[e]|.
//  2. router_select_kernel, one warp per token: |a_e - l_e| <= B_e, where l_e
//     is the canonical logit and B_e = d 2^-21 |x_t| |W_r[e]| + 2^-20 (|a_e| +
//     |bias_e|) + 2^-100, the norms (fp32) and the sum each inflated by 2^-8
//     (every sum of d exact products in
//     fp32 with round-to-nearest or truncation is within (d - 1) 2^-23
//     sum |x_i w_i| <= (d - 1) 2^-23 |x| |w| of the exact sum, by
//     Cauchy-Schwarz: the bound allows four times that for the tensor cores'
//     unspecified accumulation order, plus the rounding of the bias add). With
//     L the k-th largest lower bound a_e - B_e, at least k experts have
//     l >= L, so an expert with a_e + B_e < L is not among the top k. The
//     remaining candidates (typically k plus a few) get their canonical logit,
//     computed exactly as the other router kernels do; non-candidates rank as
//     NaN (after every number) in the usual top-k. A token whose approximate
//     logits or norms are not finite gets every logit computed exactly.
// The result is the top-k of the canonical logits, bit for bit, and the gates
// are the softmax of the k chosen canonical logits.
#include <string.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tma.h"

namespace moe {
namespace {

constexpr int kRaStages = 4;
constexpr int kRaThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue (or, in a norm CTA, all six)
constexpr int kRaTile = 128;     // tokens per CTA (M)
constexpr int kRaN = 64;         // experts per CTA (N): 4 x 32 CTAs for 4096 tokens and 256 experts
constexpr int kRaRowBytes = 128; // K per stage: 64 bf16 = one 128-byte swizzled row

struct RaArgs {
    CUtensorMap mx, mw;     // x [T][d] in 128 x 64 boxes, W_r [E][d] in 64 x 64 boxes, 128-byte swizzled
    const uint16_t *wr;
    const float *bias;
    int T, E, d;
    float *approx;          // [T][E]
    float *wnorm;           // [E]
    int *err;
};

struct RaSmem {
    uint8_t x[kRaStages][kRaTile * kRaRowBytes];
    uint8_t w[kRaStages][kRaN * kRaRowBytes];
    uint64_t full[kRaStages], empty[kRaStages], acc_full;
    uint32_t tmem_base;
};
constexpr int kRaSmemBytes = (int)sizeof(RaSmem) + 1024;

__device__ __forceinline__ RaSmem &ra_smem(uint8_t *raw) {
    return *reinterpret_cast<RaSmem *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
}

__global__ void __launch_bounds__(kRaThreads, 1) router_approx_kernel(const __grid_constant__ RaArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (blockIdx.x == gridDim.x - 1) {
        // norm CTA: |W_r[e]| (fp32 sum of squares) for experts 64 y .. 64 y + 63
        const int e1 = min(a.E, (int)(blockIdx.y + 1) * kRaN);
        for (int e = blockIdx.y * kRaN + warp; e < e1; e += kRaThreads / 32) {
            const uint16_t *r = a.wr + (int64_t)e * a.d;
            float ss = 0.f;
            for (int i = 8 * lane; i < a.d; i += 256) {
                const uint4 v = __ldg(reinterpret_cast<const uint4 *>(r + i));
                const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float lo = __uint_as_float(u[j] << 16), hi = __uint_as_float(u[j] & 0xFFFF0000u);
                    ss = fmaf(lo, lo, fmaf(hi, hi, ss));
                }
            }
            ss = warp_sum(ss);
            if (lane == 0) a.wnorm[e] = sqrtf(ss);
        }
        return;
    }
    extern __shared__ uint8_t smem_raw[];
    RaSmem &s = ra_smem(smem_raw);
    if (threadIdx.x == 0) {
        for (int i = 0; i < kRaStages; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1);
        }
        mbar_init(&s.acc_full, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&s.tmem_base, kRaN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;
    const int t0 = blockIdx.x * kRaTile, e0 = blockIdx.y * kRaN, nk = a.d / 64;
    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&a.mx);
            prefetch_tensormap(&a.mw);
            int kt = 0;
            for (; kt < nk; ++kt) {
                const int slot = kt % kRaStages;
                if (!mbar_wait(&s.empty[slot], ((kt / kRaStages) & 1) ^ 1)) {
                    set_device_error(a.err, MOE_DEVERR_TIMEOUT);
                    break;
                }
                mbar_arrive_expect_tx(&s.full[slot], (kRaTile + kRaN) * kRaRowBytes);
                tma_load_2d(s.x[slot], &a.mx, kt * kRaRowBytes, t0, &s.full[slot]);
                tma_load_2d(s.w[slot], &a.mw, kt * kRaRowBytes, e0, &s.full[slot]);
            }
            for (int g = kt - kRaStages; g < kt; ++g)  // copies in flight land before the CTA exits
                if (g >= 0) mbar_wait(&s.full[g % kRaStages], (g / kRaStages) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(kRaTile, kRaN);
            bool ok = true;
            for (int kt = 0; kt < nk; ++kt) {
                const int slot = kt % kRaStages;
                if (!mbar_wait(&s.full[slot], (kt / kRaStages) & 1)) { ok = false; break; }
                tc_fence_after();
                const uint64_t dx = sdesc_sw128(s.x[slot]), dw = sdesc_sw128(s.w[slot]);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)  // K = 16 bf16 (32 bytes) per MMA
                    tc_mma_bf16(tmem, dx + 2 * ks, dw + 2 * ks, idesc, (kt | ks) != 0);
                tc_commit(&s.empty[slot]);
            }
            if (!ok) set_device_error(a.err, MOE_DEVERR_TIMEOUT);
            tc_commit(&s.acc_full);  // also when cut short: the epilogue must not wait forever
            mbar_wait(&s.acc_full, 0);  // every MMA done before tensor memory is freed
        }
    } else {
        // TMEM lane = token of the tile, column = expert of the tile
        const int q = warp & 3;
        const int t = t0 + 32 * q + lane;
        const bool ok = mbar_wait(&s.acc_full, 0);
        tc_fence_after();
        if (__all_sync(0xffffffffu, ok)) {
            const uint32_t base = tmem + ((uint32_t)(32 * q) << 16);
            for (int c0 = 0; c0 < kRaN; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(base + c0, v);
                tmem_wait_ld();
                if (t < a.T) {
                    float *dst = a.approx + (int64_t)t * a.E;
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int e = e0 + c0 + c;
                        if (e < a.E) dst[e] = __uint_as_float(v[c]) + (a.bias ? a.bias[e] : 0.f);
                    }
                }
            }
        } else if (lane == 0) {
            set_device_error(a.err, MOE_DEVERR_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kRaN);
    }
}

// Canonical logit of (x row, router row): lane c runs the fma chain over
// chunk c in element order, then the butterfly; every lane returns the sum.
__device__ __forceinline__ float canonical_dot(const uint16_t *xr, const uint16_t *wrow, int chunk, int lane) {
    const uint4 *xp = reinterpret_cast<const uint4 *>(xr + lane * chunk);
    const uint4 *wp = reinterpret_cast<const uint4 *>(wrow + lane * chunk);
    float acc = 0.f;
#pragma unroll 4
    for (int v = 0; v < chunk / 8; ++v) {
        const uint4 xv = __ldg(xp + v), wv = __ldg(wp + v);
        const uint32_t xa[4] = {xv.x, xv.y, xv.z, xv.w}, wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            acc = __fmaf_rn(__uint_as_float(xa[j] << 16), __uint_as_float(wa[j] << 16), acc);
            acc = __fmaf_rn(__uint_as_float(xa[j] & 0xFFFF0000u), __uint_as_float(wa[j] & 0xFFFF0000u), acc);
        }
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
    return acc;
}

constexpr int kSelWarps = 4;   // tokens per CTA
constexpr int kSelSlots = 3;   // router rows in flight per warp

struct SelArgs {
    CUtensorMap mw;  // W_r as [E d / 64][128 bytes]: one router row = one box of d / 64 rows
    const uint16_t *x, *wr;
    const float *bias, *approx, *wnorm;
    int T, d, E, k;
    int32_t *idx;
    float *gates;
    int *err;
};

// One warp per token; lane holds experts lane + 32 i (NC = E / 32 rounded up).
// RB > 0 (d = 64 RB, 2048 or 4096): the token's x chunk stays in registers and
// each candidate's router row comes into shared memory as one TMA box (rows
// of 128 bytes, 128-byte swizzled; lane c's chunk is box rows c RB / 32 ..),
// kSelSlots rows in flight per warp, so the rows cross from L2 in whole lines
// and the lanes read their chunks with few bank conflicts. RB = 0: any d, each
// lane reads its chunk from global memory, one candidate at a time.
template <int NC, int RB>
__global__ void __launch_bounds__(kSelWarps * 32) router_select_kernel(const __grid_constant__ SelArgs a) {
    constexpr int NV = RB > 0 ? RB / 4 : 1;      // uint4 of x per lane (chunk = d / 32 = 2 RB elements)
    constexpr int kRow = RB > 0 ? RB * 128 : 0;   // bytes of one router row
    __shared__ float sl[kSelWarps][NC * 32];
    __shared__ int16_t scand[kSelWarps][NC * 32];
    __shared__ uint64_t sbar[kSelWarps][kSelSlots];
    extern __shared__ uint8_t sel_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kSelWarps + warp;
    if (t >= a.T) return;
    const int d = a.d, E = a.E, k = a.k;
    float *lw = sl[warp];
    // 128-byte-swizzled boxes need 1024-byte aligned destinations (1 KB of slack is allocated)
    uint8_t *wbuf = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sel_raw) + 1023) & ~uintptr_t(1023)) +
                    (size_t)warp * kSelSlots * (kRow > 0 ? kRow : 1);
    if (RB > 0 && lane == 0) {
        for (int i = 0; i < kSelSlots; ++i) mbar_init(&sbar[warp][i], 1);
        fence_mbar_init();
    }
    const uint16_t *xr = a.x + (int64_t)t * d;
    const int chunk = d / 32;
    uint4 xv[NV];
    if (RB > 0)
#pragma unroll
        for (int v = 0; v < NV; ++v) xv[v] = __ldg(reinterpret_cast<const uint4 *>(xr + lane * chunk) + v);
    float ss = 0.f;  // |x_t|^2
    if (RB > 0) {
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const uint32_t w[4] = {xv[v].x, xv[v].y, xv[v].z, xv[v].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float lo = __uint_as_float(w[j] << 16), hi = __uint_as_float(w[j] & 0xFFFF0000u);
                ss = fmaf(lo, lo, fmaf(hi, hi, ss));
            }
        }
    } else {
        for (int v = 0; v < chunk / 8; ++v) {
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(xr + lane * chunk) + v);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float lo = __uint_as_float(w[j] << 16), hi = __uint_as_float(w[j] & 0xFFFF0000u);
                ss = fmaf(lo, lo, fmaf(hi, hi, ss));
            }
        }
    }
    const float nx = sqrtf(warp_sum(ss)) * (1.0f + 0x1p-8f);  // fp32 norms, inflated past their rounding
    const float gam = (float)d * 0x1p-21f;
    float av[NC], bnd[NC];
    bool bad = !isfinite(nx);
#pragma unroll
    for (int i = 0; i < NC; ++i) {
        const int e = lane + 32 * i;
        av[i] = 0.f;
        bnd[i] = 0.f;
        if (e < E) {
            av[i] = a.approx[(int64_t)t * E + e];
            const float b = a.bias ? fabsf(a.bias[e]) : 0.f;
            bnd[i] = (gam * nx * (a.wnorm[e] * (1.0f + 0x1p-8f)) + 0x1p-20f * (fabsf(av[i]) + b) + 0x1p-100f) *
                     (1.0f + 0x1p-8f);
            bad |= !isfinite(av[i]) || !isfinite(bnd[i]);
        }
    }
    bad = __any_sync(0xffffffffu, bad);
    float L = 0.f;
    if (!bad) {  // L = the k-th largest lower bound
        float lb[NC];
#pragma unroll
        for (int i = 0; i < NC; ++i) {
            lb[i] = av[i] - bnd[i];
            if (lane + 32 * i < E) lw[lane + 32 * i] = lb[i];
        }
        __syncwarp();
        const int pk = topk_warp<NC>(lb, E, k, lane);
        const int ek = __shfl_sync(0xffffffffu, pk, k - 1);
        L = lw[ek];
        __syncwarp();
    }
    // canonical logits of the candidates; the others rank as NaN (last)
    int nc = 0;
#pragma unroll
    for (int i = 0; i < NC; ++i) {
        const int e = lane + 32 * i;
        const bool cand = e < E && (bad || av[i] + bnd[i] >= L);
        if (e < E && !cand) lw[e] = __uint_as_float(0x7FC00000u);
        const unsigned m = __ballot_sync(0xffffffffu, cand);
        if (cand) scand[warp][nc + __popc(m & ((1u << lane) - 1u))] = (int16_t)e;
        nc += __popc(m);
    }
    __syncwarp();
    if (RB > 0) {
        auto fetch = [&](int c) {  // candidate c's router row into slot c % kSelSlots
            uint64_t *bar = &sbar[warp][c % kSelSlots];
            mbar_arrive_expect_tx(bar, kRow);
            tma_load_2d(wbuf + (size_t)(c % kSelSlots) * kRow, &a.mw, 0, (int)scand[warp][c] * RB, bar);
        };
        if (lane == 0)
            for (int c = 0; c < min(nc, kSelSlots); ++c) fetch(c);
        for (int c = 0; c < nc; ++c) {
            const int slot = c % kSelSlots;
            if (!mbar_wait(&sbar[warp][slot], (c / kSelSlots) & 1)) {
                set_device_error(a.err, MOE_DEVERR_TIMEOUT);
                // the copies issued after c must land before the warp leaves
                for (int g = c + 1; g < min(nc, c + kSelSlots); ++g)
                    mbar_wait(&sbar[warp][g % kSelSlots], (g / kSelSlots) & 1);
                break;
            }
            const uint8_t *row = wbuf + (size_t)slot * kRow;
            float acc = 0.f;
#pragma unroll
            for (int v = 0; v < NV; ++v) {  // chunk element order: box row lane RB / 32 + v / 8, unit v % 8
                const int r = lane * (RB / 32) + (v >> 3), u = v & 7;
                const uint4 wv = lds128(row + r * 128 + (((u ^ (r & 7))) << 4));
                const uint32_t xa[4] = {xv[v].x, xv[v].y, xv[v].z, xv[v].w}, wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc = __fmaf_rn(__uint_as_float(xa[j] << 16), __uint_as_float(wa[j] << 16), acc);
                    acc = __fmaf_rn(__uint_as_float(xa[j] & 0xFFFF0000u), __uint_as_float(wa[j] & 0xFFFF0000u), acc);
                }
            }
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
            const int ee = scand[warp][c];
            if (lane == 0) lw[ee] = a.bias ? __fadd_rn(acc, a.bias[ee]) : acc;
            __syncwarp();  // every lane's reads of the slot are done before it is refilled
            if (lane == 0 && c + kSelSlots < nc) {
                fence_proxy_async_smem();
                fetch(c + kSelSlots);
            }
        }
    } else {
        for (int c = 0; c < nc; ++c) {
            const int ee = scand[warp][c];
            float v = canonical_dot(xr, a.wr + (int64_t)ee * d, chunk, lane);
            if (a.bias) v = __fadd_rn(v, a.bias[ee]);
            if (lane == 0) lw[ee] = v;
        }
    }
    __syncwarp();
    float cv[NC];
#pragma unroll
    for (int i = 0; i < NC; ++i) cv[i] = lane + 32 * i < E ? lw[lane + 32 * i] : 0.f;
    const int my_e = topk_warp<NC>(cv, E, k, lane);
    const float my_l = lane < k ? lw[my_e] : 0.f;
    const float l0 = __shfl_sync(0xffffffffu, my_l, 0);
    const float ex = lane < k ? expf(my_l - l0) : 0.f;
    const float den = warp_sum(ex);
    if (lane < k) {
        a.idx[(int64_t)t * k + lane] = my_e;
        a.gates[(int64_t)t * k + lane] = ex / den;
    }
}

}  // namespace

bool router_tc_applies(const moe_dims &d) {
    return d.route == MOE_ROUTE_SOFTMAX_TOPK && d.T >= 32 && d.d_model % 64 == 0 && d.E <= 1024;
}

cudaError_t launch_router_approx(const moe_dims &d, const uint16_t *x, const moe_weights &w, float *approx,
                                 float *wnorm, cudaStream_t s) {
    static std::atomic<bool> attr[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(router_approx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kRaSmemBytes);
        if (e != cudaSuccess) return e;
        attr[dev].store(true, std::memory_order_release);
    }
    RaArgs a;
    memset(&a, 0, sizeof a);
    if (!make_tile_map_u8(&a.mx, x, d.T, (uint64_t)d.d_model * 2, kRaTile) ||
        !make_tile_map_u8(&a.mw, w.w_router, d.E, (uint64_t)d.d_model * 2, kRaN))
        return cudaErrorInvalidValue;
    a.wr = w.w_router;
    a.bias = w.router_bias;
    a.T = d.T; a.E = d.E; a.d = d.d_model;
    a.approx = approx;
    a.wnorm = wnorm;
    a.err = device_error_word();
    const dim3 grid(ceil_div(d.T, kRaTile) + 1, ceil_div(d.E, kRaN));
    router_approx_kernel<<<grid, kRaThreads, kRaSmemBytes, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_route_tc(const moe_dims &d, const uint16_t *x, const moe_weights &w, int32_t *idx, float *gates,
                            float *approx, float *wnorm, cudaStream_t s) {
    cudaError_t e = launch_router_approx(d, x, w, approx, wnorm, s);
    if (e != cudaSuccess) return e;
    SelArgs sa;
    memset(&sa, 0, sizeof sa);
    sa.x = x; sa.wr = w.w_router; sa.bias = w.router_bias; sa.approx = approx; sa.wnorm = wnorm;
    sa.T = d.T; sa.d = d.d_model; sa.E = d.E; sa.k = d.k; sa.idx = idx; sa.gates = gates;
    sa.err = device_error_word();
    const dim3 grid(ceil_div(d.T, kSelWarps));
    const int rb = d.d_model / 64;
    if (d.E <= 256 && (rb == 64 || rb == 32)) {
        if (!make_tile_map_u8(&sa.mw, w.w_router, (uint64_t)d.E * rb, 128, (uint32_t)rb)) return cudaErrorInvalidValue;
        const size_t smem = (size_t)kSelWarps * kSelSlots * rb * 128 + 1024;
        auto kern = rb == 64 ? router_select_kernel<8, 64> : router_select_kernel<8, 32>;
        static std::atomic<bool> attr[64];
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
        if (!attr[dev].load(std::memory_order_acquire)) {
            for (int r : {64, 32}) {
                cudaError_t e2 = cudaFuncSetAttribute(r == 64 ? router_select_kernel<8, 64> : router_select_kernel<8, 32>,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                      kSelWarps * kSelSlots * r * 128 + 1024);
                if (e2 != cudaSuccess) return e2;
            }
            attr[dev].store(true, std::memory_order_release);
        }
        kern<<<grid, kSelWarps * 32, smem, s>>>(sa);
    } else if (d.E <= 256) {
        router_select_kernel<8, 0><<<grid, kSelWarps * 32, 0, s>>>(sa);
    } else {
        router_select_kernel<32, 0><<<grid, kSelWarps * 32, 0, s>>>(sa);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
