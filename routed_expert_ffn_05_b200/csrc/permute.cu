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

// Block b counts the experts of slots [b*256, b*256 + 256).
__global__ void __launch_bounds__(kPermuteBlock) permute_hist_kernel(const int32_t *__restrict__ idx,
                                                                     int64_t S, int E,
                                                                     int32_t *__restrict__ blkcnt, int *err) {
    extern __shared__ int32_t hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int64_t s = (int64_t)blockIdx.x * kPermuteBlock + threadIdx.x;
    if (s < S) {
        const int e = idx[s];
        if (e < 0 || e >= E) set_device_error(err, MOE_DEVERR_EXPERT_RANGE);
        else atomicAdd(&hist[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) blkcnt[(int64_t)blockIdx.x * E + e] = hist[e];
}

// One block: per-expert totals over blocks, the exclusive scan over experts,
// then blkbase[b][e] = the first row of block b's slots of expert e. Thread e
// reads its column of block counts 16 at a time (independent loads in flight).
__global__ void __launch_bounds__(1024) permute_scan_kernel(const int32_t *__restrict__ blkcnt,
                                                            int64_t nblk, int E,
                                                            int32_t *__restrict__ blkbase,
                                                            int32_t *__restrict__ counts,
                                                            int32_t *__restrict__ offsets) {
    __shared__ int32_t sc[1024];
    constexpr int kBatch = 16;
    const int e = threadIdx.x;
    int32_t run = 0;
    if (e < E)
        for (int64_t b0 = 0; b0 < nblk; b0 += kBatch) {
            int32_t c[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) c[j] = b0 + j < nblk ? blkcnt[(b0 + j) * E + e] : 0;
#pragma unroll
            for (int j = 0; j < kBatch; ++j) run += c[j];
        }
    sc[e] = e < E ? run : 0;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {  // inclusive Hillis-Steele scan
        const int32_t v = e >= o ? sc[e - o] : 0;
        __syncthreads();
        sc[e] += v;
        __syncthreads();
    }
    if (e < E) {
        const int32_t excl = sc[e] - run;
        counts[e] = run;
        offsets[e] = excl;
        if (e == E - 1) offsets[E] = sc[e];
        int32_t r = excl;
        for (int64_t b0 = 0; b0 < nblk; b0 += kBatch) {
            int32_t c[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) c[j] = b0 + j < nblk ? blkcnt[(b0 + j) * E + e] : 0;
#pragma unroll
            for (int j = 0; j < kBatch; ++j)
                if (b0 + j < nblk) {
                    blkbase[(b0 + j) * E + e] = r;
                    r += c[j];
                }
        }
    }
}

__global__ void __launch_bounds__(kPermuteBlock) permute_scatter_kernel(
    const int32_t *__restrict__ idx, int64_t S, int E, const int32_t *__restrict__ blkbase,
    int32_t *__restrict__ perm, int32_t *__restrict__ inv_perm) {
    extern __shared__ int32_t wcnt[];  // [kWarps][E]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    const int64_t s = (int64_t)blockIdx.x * kPermuteBlock + threadIdx.x;
    int e = -1;
    if (s < S) {
        e = idx[s];
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
    }
}

cudaError_t launch_permute(const moe_dims &d, const int32_t *idx, int32_t *counts, int32_t *offsets,
                           int32_t *perm, int32_t *inv_perm, int32_t *blkcnt, int32_t *blkbase,
                           int64_t nblk, cudaStream_t s) {
    const int64_t S = (int64_t)d.T * d.k;
    if (nblk > 0)
        permute_hist_kernel<<<(unsigned)nblk, kPermuteBlock, d.E * 4, s>>>(idx, S, d.E, blkcnt,
                                                                           device_error_word());
    permute_scan_kernel<<<1, 1024, 0, s>>>(blkcnt, nblk, d.E, blkbase, counts, offsets);
    if (nblk > 0)
        permute_scatter_kernel<<<(unsigned)nblk, kPermuteBlock, kWarps * d.E * 4, s>>>(idx, S, d.E, blkbase,
                                                                                      perm, inv_perm);
    count_launches(nblk > 0 ? 3 : 1);
    return cudaGetLastError();
}

}  // namespace moe
