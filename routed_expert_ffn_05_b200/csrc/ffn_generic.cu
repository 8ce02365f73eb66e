// Generic expert FFN on CUDA cores: any T, any weight format and activation
// mode. One warp per (permuted row, output feature), dequantisation fused into
// the dot product. It is the reference-shaped path for shapes the specialised
// kernels do not cover.
//
// Each expert is a SwiGLU FFN, h = silu(W1 a) * (W3 a), o = W2 h; the routed
// experts are block-quantised, the shared expert is bf16 ("DS4", dibi8.com,
// "Key architectural innovations" item 1; "DwarfStar", hysenlabs.com, "Model
// support and quantisation"). In bf16-activation mode h is rounded to bf16
// before W2; in MXFP8 (MXFP4) mode x and h are quantised to MXFP8 (MXFP4)
// along their length.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

struct ActRow {  // one activation row: bf16, fp32 (bf16-valued), MXFP8 or MXFP4
    const uint16_t *bf;
    const float *f;
    const uint8_t *codes;   // E4M3, one per byte
    const uint8_t *scales;
    const uint8_t *codes4;  // E2M1, two per byte (element 2i in the low nibble)
    __device__ __forceinline__ float operator()(int i) const {
        if (bf) return bf16_to_f32(bf[i]);
        if (f) return f[i];
        if (codes4) return e2m1_to_f32((codes4[i / 2] >> (4 * (i & 1))) & 15u) * e8m0_to_f32(scales[i / 32]);
        const __half_raw h = __nv_cvt_fp8_to_halfraw(codes[i], __NV_E4M3);
        return __half2float(__half(h)) * e8m0_to_f32(scales[i / 32]);
    }
};

// sum over the 32 elements of block kb of a(i) * W[row][i].
__device__ __forceinline__ float block_dot(int wfmt, const uint8_t *packed, int64_t off_a, int64_t off_b,
                                           int64_t off_c, int64_t row, int K, int kb, const ActRow &a) {
    float acc = 0.0f;
    if (wfmt == MOE_W_Q2K) {
        const int64_t sb = row * (K / 256) + kb / 8;
        const uint32_t dd = reinterpret_cast<const uint32_t *>(packed + off_c)[sb];
        const float dv = __half2float(__ushort_as_half((uint16_t)(dd & 0xFFFF)));
        const float mv = __half2float(__ushort_as_half((uint16_t)(dd >> 16)));
        const uint32_t *qw = reinterpret_cast<const uint32_t *>(packed + off_a) + sb * 16;
        for (int h = 0; h < 2; ++h) {
            const uint8_t scm = packed[off_b + sb * 16 + (kb % 8) * 2 + h];
            const float ds = __fmul_rn(dv, (float)(scm & 15)), dm = __fmul_rn(mv, (float)(scm >> 4));
            for (int j = 0; j < 16; ++j) {
                const int e = (kb % 8) * 32 + 16 * h + j;  // quant index in the super-block
                const int qq = (int)((qw[q2k_word(e)] >> q2k_bit(e)) & 3u);
                acc = fmaf(a(kb * 32 + 16 * h + j), __fsub_rn(__fmul_rn(ds, (float)qq), dm), acc);
            }
        }
        return acc;
    }
    const uint4 c = reinterpret_cast<const uint4 *>(packed + off_a + row * (K / 2))[kb];
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 32; ++i) acc = fmaf(a(kb * 32 + i), e2m1_to_f32((w[i / 8] >> (4 * (i % 8))) & 15u), acc);
    return acc * e8m0_to_f32(packed[off_b + row * (K / 32) + kb]);
}

struct MatRef {
    const uint8_t *p;
    int64_t a, b, c;
};
static MatRef mat_ref(const moe_dims &d, int which, const void *packed) {
    MatRef m;
    m.p = static_cast<const uint8_t *>(packed);
    if (d.wfmt == MOE_W_Q2K) {
        const Q2kLayout L = q2k_layout(d, which);
        m.a = L.qs; m.b = L.scm; m.c = L.dd;
    } else {
        const Mxfp4Layout L = mxfp4_layout(d, which);
        m.a = L.codes; m.b = L.srow; m.c = 0;
    }
    return m;
}

__global__ void __launch_bounds__(256) gateup_generic_kernel(moe_dims d, MatRef w1, MatRef w3,
                                                             const uint16_t *__restrict__ x,
                                                             const uint8_t *__restrict__ x8,
                                                             const uint8_t *__restrict__ xs,
                                                             const int32_t *__restrict__ offsets,
                                                             const int32_t *__restrict__ perm,
                                                             float *__restrict__ h) {
    const int r = blockIdx.x, n = blockIdx.y * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (n >= d.d_ff) return;
    const int e = expert_of_row(offsets, d.E, r);
    const int t = perm[r] / d.k;
    const int K = d.d_model;
    ActRow a{nullptr, nullptr, nullptr, nullptr, nullptr};
    if (d.act == MOE_A_MXFP8) { a.codes = x8 + (int64_t)t * K; a.scales = xs + (int64_t)t * (K / 32); }
    else if (d.act == MOE_A_MXFP4) { a.codes4 = x8 + (int64_t)t * (K / 2); a.scales = xs + (int64_t)t * (K / 32); }
    else a.bf = x + (int64_t)t * K;
    const int64_t row = (int64_t)e * d.d_ff + n;
    float g = 0.0f, u = 0.0f;
    for (int kb = lane; kb < K / 32; kb += 32) {
        g += block_dot(d.wfmt, w1.p, w1.a, w1.b, w1.c, row, K, kb, a);
        u += block_dot(d.wfmt, w3.p, w3.a, w3.b, w3.c, row, K, kb, a);
    }
    g = warp_sum(g);
    u = warp_sum(u);
    if (lane == 0) {
        float hv = silu_f32(g) * u;
        if (d.act == MOE_A_BF16) hv = bf16_to_f32(f32_to_bf16_rne(hv));
        h[(int64_t)r * d.d_ff + n] = hv;
    }
}

__global__ void __launch_bounds__(256) down_generic_kernel(moe_dims d, MatRef w2, const float *__restrict__ h,
                                                           const uint8_t *__restrict__ h8,
                                                           const uint8_t *__restrict__ hs,
                                                           const int32_t *__restrict__ offsets,
                                                           float *__restrict__ out) {
    const int r = blockIdx.x, i = blockIdx.y * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (i >= d.d_model) return;
    const int e = expert_of_row(offsets, d.E, r);
    const int K = d.d_ff;
    ActRow a{nullptr, nullptr, nullptr, nullptr, nullptr};
    if (d.act == MOE_A_MXFP8) { a.codes = h8 + (int64_t)r * K; a.scales = hs + (int64_t)r * (K / 32); }
    else if (d.act == MOE_A_MXFP4) { a.codes4 = h8 + (int64_t)r * (K / 2); a.scales = hs + (int64_t)r * (K / 32); }
    else a.f = h + (int64_t)r * K;
    const int64_t row = (int64_t)e * d.d_model + i;
    float o = 0.0f;
    for (int kb = lane; kb < K / 32; kb += 32) o += block_dot(d.wfmt, w2.p, w2.a, w2.b, w2.c, row, K, kb, a);
    o = warp_sum(o);
    if (lane == 0) out[(int64_t)r * d.d_model + i] = o;
}

cudaError_t launch_expert_ffn_generic(const moe_dims &d, const moe_weights &w, const uint16_t *x,
                                      const int32_t *offsets, const int32_t *perm, float *out_rows,
                                      uint8_t *ws, const WsLayout &L, cudaStream_t s) {
    const int64_t S = (int64_t)d.T * d.k;
    if (S == 0) return cudaSuccess;
    uint8_t *x8 = ws + L.x8, *xs = ws + L.xs, *h8 = ws + L.h8, *hs = ws + L.hs;
    float *h = reinterpret_cast<float *>(ws + L.h);
    cudaError_t err;
    const bool q = d.act != MOE_A_BF16, fp4 = d.act == MOE_A_MXFP4;
    if (q && (err = launch_quant_act_bf16(x, d.T, d.d_model, x8, xs, s, fp4)) != cudaSuccess) return err;
    gateup_generic_kernel<<<dim3((unsigned)S, ceil_div(d.d_ff, 8)), 256, 0, s>>>(
        d, mat_ref(d, MOE_MAT_W1, w.w1), mat_ref(d, MOE_MAT_W3, w.w3), x, x8, xs, offsets, perm, h);
    if (q && (err = launch_quant_act_f32(h, S, d.d_ff, h8, hs, s, fp4)) != cudaSuccess) return err;
    down_generic_kernel<<<dim3((unsigned)S, ceil_div(d.d_model, 8)), 256, 0, s>>>(
        d, mat_ref(d, MOE_MAT_W2, w.w2), h, h8, hs, offsets, out_rows);
    count_launches(2);
    return cudaGetLastError();
}

// Shared expert: bf16 weights and activations, h rounded to bf16.
__global__ void __launch_bounds__(256) shared_gateup_kernel(const uint16_t *__restrict__ x,
                                                            const uint16_t *__restrict__ w1,
                                                            const uint16_t *__restrict__ w3, int d, int Fs,
                                                            float *__restrict__ h) {
    const int t = blockIdx.x, n = blockIdx.y * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (n >= Fs) return;
    const uint16_t *xr = x + (int64_t)t * d, *a = w1 + (int64_t)n * d, *b = w3 + (int64_t)n * d;
    float g = 0.0f, u = 0.0f;
    for (int i = lane; i < d; i += 32) {
        const float xv = bf16_to_f32(xr[i]);
        g = fmaf(xv, bf16_to_f32(a[i]), g);
        u = fmaf(xv, bf16_to_f32(b[i]), u);
    }
    g = warp_sum(g);
    u = warp_sum(u);
    if (lane == 0) h[(int64_t)t * Fs + n] = bf16_to_f32(f32_to_bf16_rne(silu_f32(g) * u));
}

__global__ void __launch_bounds__(256) shared_down_kernel(const float *__restrict__ h,
                                                          const uint16_t *__restrict__ w2, int d, int Fs,
                                                          float *__restrict__ out) {
    const int t = blockIdx.x, i = blockIdx.y * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (i >= d) return;
    const float *hr = h + (int64_t)t * Fs;
    const uint16_t *wr = w2 + (int64_t)i * Fs;
    float o = 0.0f;
    for (int f = lane; f < Fs; f += 32) o = fmaf(hr[f], bf16_to_f32(wr[f]), o);
    o = warp_sum(o);
    if (lane == 0) out[(int64_t)t * d + i] = o;
}

cudaError_t launch_shared_ffn_generic(const moe_dims &d, const moe_weights &w, const uint16_t *x,
                                      float *out, float *hbuf, cudaStream_t s) {
    if (d.T == 0) return cudaSuccess;
    shared_gateup_kernel<<<dim3(d.T, ceil_div(d.d_ff_shared, 8)), 256, 0, s>>>(x, w.sw1, w.sw3, d.d_model,
                                                                                d.d_ff_shared, hbuf);
    shared_down_kernel<<<dim3(d.T, ceil_div(d.d_model, 8)), 256, 0, s>>>(hbuf, w.sw2, d.d_model,
                                                                          d.d_ff_shared, out);
    count_launches(2);
    return cudaGetLastError();
}

cudaError_t launch_expert_ffn(const moe_dims &d, const moe_weights &w, const uint16_t *x,
                              const int32_t *offsets, const int32_t *perm, float *out_rows, float *shared_out,
                              uint8_t *ws, const WsLayout &L, cudaStream_t s, bool prepared, bool rows_bf16) {
    if (decode_path_applies(d))
        return launch_decode_ffn(d, w, x, offsets, perm, out_rows, shared_out, ws, L, s, prepared);
    cudaError_t e;
    if (shared_out &&
        (e = launch_shared_ffn_generic(d, w, x, shared_out, reinterpret_cast<float *>(ws + L.sh_h), s)) != cudaSuccess)
        return e;
    if (tc_path_applies(d)) return launch_tc_ffn(d, w, x, offsets, perm, out_rows, ws, L, s, rows_bf16);
    if (tc16_path_applies(d)) return launch_tc16_ffn(d, w, x, offsets, perm, out_rows, ws, L, s);
    return launch_expert_ffn_generic(d, w, x, offsets, perm, out_rows, ws, L, s);
}

cudaError_t launch_shared_ffn(const moe_dims &d, const moe_weights &w, const uint16_t *x, float *out,
                              float *hbuf, cudaStream_t s) {
    return launch_shared_ffn_generic(d, w, x, out, hbuf, s);
}

}  // namespace moe
