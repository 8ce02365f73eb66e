// Gate-weighted combine: y[t] = sum_{j ascending} w[t,j] * o[inv_perm[t*k+j]]
// (+ shared expert s[t]), fp32, the k terms in a fixed order. A slot whose
// inv_perm entry is negative (no valid expert) is skipped. With `accumulate`
// the sum is added to y instead (later waves of the expert cache). The expert
// rows o are fp32 (the staged API) or bf16 (the fused layer's w4a8 path,
// which halves their write and read traffic).
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {

__device__ __forceinline__ float4 load_row4(const float *r, int i4) { return reinterpret_cast<const float4 *>(r)[i4]; }
__device__ __forceinline__ float4 load_row4(const uint16_t *r, int i4) {
    const uint2 v = reinterpret_cast<const uint2 *>(r)[i4];
    return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u), __uint_as_float(v.y << 16),
                       __uint_as_float(v.y & 0xFFFF0000u));
}

template <typename R>
__global__ void __launch_bounds__(256) combine_kernel(const R *__restrict__ out_rows,
                                                      const int32_t *__restrict__ inv_perm,
                                                      const float *__restrict__ gates,
                                                      const float *__restrict__ shared, int d, int k,
                                                      float *__restrict__ y, int accumulate) {
    grid_dep_wait();  // launched programmatically after the expert FFN: its outputs first
    const int t = blockIdx.y;
    const int i4 = blockIdx.x * blockDim.x + threadIdx.x;  // float4 index
    if (i4 * 4 >= d) return;
    float4 acc = accumulate ? reinterpret_cast<const float4 *>(y + (int64_t)t * d)[i4]
                 : shared   ? reinterpret_cast<const float4 *>(shared + (int64_t)t * d)[i4]
                            : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
        const int64_t s = (int64_t)t * k + j;
        const int row = inv_perm[s];
        if (row < 0) continue;  // a slot without an expert (its error is already reported) adds nothing
        const float g = gates[s];
        const float4 o = load_row4(out_rows + (int64_t)row * d, i4);
        sum.x = fmaf(g, o.x, sum.x);
        sum.y = fmaf(g, o.y, sum.y);
        sum.z = fmaf(g, o.z, sum.z);
        sum.w = fmaf(g, o.w, sum.w);
    }
    acc.x += sum.x;
    acc.y += sum.y;
    acc.z += sum.z;
    acc.w += sum.w;
    reinterpret_cast<float4 *>(y + (int64_t)t * d)[i4] = acc;
}

template <typename R>
static cudaError_t launch_combine_t(const moe_dims &d, const R *out_rows, const int32_t *inv_perm,
                                   const float *gates, const float *shared, float *y, cudaStream_t s, bool pdl,
                                   bool accumulate) {
    if (d.T == 0) return cudaSuccess;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ceil_div(d.d_model / 4, 256), d.T);
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    const int dm = d.d_model, k = d.k, acc = accumulate ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, combine_kernel<R>, out_rows, inv_perm, gates, shared, dm, k, y, acc);
    count_launches(1);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_combine(const moe_dims &d, const float *out_rows, const int32_t *inv_perm,
                           const float *gates, const float *shared, float *y, cudaStream_t s, bool pdl,
                           bool accumulate) {
    return launch_combine_t(d, out_rows, inv_perm, gates, shared, y, s, pdl, accumulate);
}

cudaError_t launch_combine_bf16(const moe_dims &d, const uint16_t *out_rows, const int32_t *inv_perm,
                                const float *gates, const float *shared, float *y, cudaStream_t s, bool accumulate) {
    return launch_combine_t(d, out_rows, inv_perm, gates, shared, y, s, false, accumulate);
}

}  // namespace moe
