// Token-by-expert histogram, exclusive scan and stable permutation.
//
// Batched expert work ("DwarfStar", hysenlabs.com, "Model support and
// quantisation") needs the slots s = t*k + j grouped by expert. Rows of one
// expert keep ascending slot order, so the result is unique and needs no
// ordering of atomics: counts come from per-block histograms, every slot's rank
// from warp match masks plus per-warp counts, all deterministic.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kWarps = kPermuteBlock / 32;

// Block b counts the experts of slots [b*256, b*256 + 256). Expert ids are
// taken relative to ebase: a slot whose id - ebase is outside [0, E) gets no
// row; it is an error (reported through err) unless err is null, which is how
// the expert-parallel layer drops the experts another rank owns.
__global__ void __launch_bounds__(kPermuteBlock) permute_hist_kernel(const int32_t *__restrict__ idx,
                                                                     int64_t S, int E, int ebase,
                                                                     int32_t *__restrict__ blkcnt, int *err) {
    extern __shared__ int32_t hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int64_t s = (int64_t)blockIdx.x * kPermuteBlock + threadIdx.x;
    if (s < S) {
        const int e = idx[s] - ebase;
        if (e < 0 || e >= E) {
            if (err) set_device_error(err, MOE_DEVERR_EXPERT_RANGE);
        } else {
            atomicAdd(&hist[e], 1);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) blkcnt[(int64_t)blockIdx.x * E + e] = hist[e];
}

// One block: per-expert totals over blocks, the exclusive scan over experts,
// then blkbase[b][e] = the first row of block b's slots of expert e. The
// 1024 threads are G = 1024 / ep groups of ep (E rounded up to a power of
// two): thread (g, e) owns expert e's counts in the g-th contiguous range of
// blocks and reads them 16 at a time, once for its partial sum and once to
// write the bases (consecutive threads read consecutive experts of a block).
__global__ void __launch_bounds__(1024) permute_scan_kernel(const int32_t *__restrict__ blkcnt,
                                                            int64_t nblk, int E,
                                                            int32_t *__restrict__ blkbase,
                                                            int32_t *__restrict__ counts,
                                                            int32_t *__restrict__ offsets) {
    __shared__ int32_t part[1024];  // [g][e]: partial sums, then the group's first row
    __shared__ int32_t sc[1024];
    constexpr int kBatch = 16;
    int ep = 1;
    while (ep < E) ep <<= 1;
    const int G = 1024 / ep, e = threadIdx.x % ep, g = threadIdx.x / ep;
    const int64_t b_lo = nblk * g / G, b_hi = nblk * (g + 1) / G;
    const bool own = e < E;
    int32_t run = 0;
    if (own)
        for (int64_t b0 = b_lo; b0 < b_hi; b0 += kBatch) {
            int32_t c[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) c[j] = b0 + j < b_hi ? blkcnt[(b0 + j) * E + e] : 0;
#pragma unroll
            for (int j = 0; j < kBatch; ++j) run += c[j];
        }
    part[threadIdx.x] = run;
    __syncthreads();
    int32_t tot = 0;  // thread i < ep: expert i's total
    if (threadIdx.x < ep)
        for (int gg = 0; gg < G; ++gg) tot += part[gg * ep + threadIdx.x];
    sc[threadIdx.x] = tot;
    __syncthreads();
    for (int o = 1; o < ep; o <<= 1) {  // inclusive Hillis-Steele scan over the experts
        const int32_t v = threadIdx.x < ep && threadIdx.x >= o ? sc[threadIdx.x - o] : 0;
        __syncthreads();
        sc[threadIdx.x] += v;
        __syncthreads();
    }
    if (threadIdx.x < E) {
        counts[threadIdx.x] = tot;
        offsets[threadIdx.x] = sc[threadIdx.x] - tot;
        if (threadIdx.x == E - 1) offsets[E] = sc[threadIdx.x];
    }
    int32_t r = 0;  // first row of this group's slots of expert e
    if (own) {
        r = e > 0 ? sc[e - 1] : 0;
        for (int gg = 0; gg < g; ++gg) r += part[gg * ep + e];
    }
    if (own)
        for (int64_t b0 = b_lo; b0 < b_hi; b0 += kBatch) {
            int32_t c[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) c[j] = b0 + j < b_hi ? blkcnt[(b0 + j) * E + e] : 0;
#pragma unroll
            for (int j = 0; j < kBatch; ++j)
                if (b0 + j < b_hi) {
                    blkbase[(b0 + j) * E + e] = r;
                    r += c[j];
                }
        }
}

__global__ void __launch_bounds__(kPermuteBlock) permute_scatter_kernel(
    const int32_t *__restrict__ idx, int64_t S, int E, int ebase, const int32_t *__restrict__ blkbase,
    int32_t *__restrict__ perm, int32_t *__restrict__ inv_perm) {
    extern __shared__ int32_t wcnt[];  // [kWarps][E]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    const int64_t s = (int64_t)blockIdx.x * kPermuteBlock + threadIdx.x;
    int e = -1;
    if (s < S) {
        e = idx[s] - ebase;
        if (e < 0 || e >= E) e = -1;
    }
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int in_warp = __popc(same & ((1u << lane) - 1u));
    if (e >= 0 && in_warp == 0) wcnt[warp * E + e] = __popc(same);
    __syncthreads();
    if (e >= 0) {
        int32_t rank = in_warp;
        for (int w = 0; w < warp; ++w) rank += wcnt[w * E + e];
        const int32_t row = blkbase[(int64_t)blockIdx.x * E + e] + rank;
        perm[row] = (int32_t)s;
        inv_perm[s] = row;
    } else if (s < S) {
        inv_perm[s] = -1;  // a slot with no valid (or no local) expert has no row
    }
}

cudaError_t launch_permute(const moe_dims &d, const int32_t *idx, int32_t *counts, int32_t *offsets,
                           int32_t *perm, int32_t *inv_perm, int32_t *blkcnt, int32_t *blkbase,
                           int64_t nblk, cudaStream_t s, int ebase, bool foreign_ok) {
    const int64_t S = (int64_t)d.T * d.k;
    if (nblk > 0)
        permute_hist_kernel<<<(unsigned)nblk, kPermuteBlock, d.E * 4, s>>>(
            idx, S, d.E, ebase, blkcnt, foreign_ok ? nullptr : device_error_word());
    permute_scan_kernel<<<1, 1024, 0, s>>>(blkcnt, nblk, d.E, blkbase, counts, offsets);
    if (nblk > 0)
        permute_scatter_kernel<<<(unsigned)nblk, kPermuteBlock, kWarps * d.E * 4, s>>>(idx, S, d.E, ebase, blkbase,
                                                                                      perm, inv_perm);
    count_launches(nblk > 0 ? 3 : 1);
    return cudaGetLastError();
}

}  // namespace moe
