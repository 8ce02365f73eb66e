// Weight quantisers (fp32 -> canonical MXFP4 / Q2_K), the packer (canonical ->
// device layout), the MXFP8 activation quantiser and a debug dequantiser.
//
// MXFP4 keeps DeepSeek's released FP4 routed-expert weights; the 2-bit build
// uses a Q2_K-style format for routed experts ("DwarfStar", hysenlabs.com,
// "Model support and quantisation"; "DS4", dibi8.com, "Key architectural
// innovations" item 1). Element and scale rules follow the OCP Microscaling
// (MX) v1.0 specification: 32-element blocks, shared scale
// 2^(floor(log2 amax) - emax_elem) stored as E8M0, elements rounded to nearest
// even and saturated. An all-zero block gets scale byte 127 and zero codes.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// Two fp32 -> packed E2M1 pair (hi in bits 4..7, lo in bits 0..3), round to
// nearest even, saturating (hardware conversion).
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float lo, float hi) {
    uint32_t out;
    asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\tcvt.u32.u8 %0, b;\n\t}"
        : "=r"(out) : "f"(hi), "f"(lo));
    return out;
}

// Shared-scale exponent of a block, clamped to the E8M0 range.
__device__ __forceinline__ int mx_shared_exp(float amax, int emax_elem) {
    int se = floor_log2_f32(amax) - emax_elem;
    return se < -127 ? -127 : (se > 127 ? 127 : se);
}

// One thread per 32-element block of fp32 weights [rows][K].
__global__ void quantize_mxfp4_kernel(const float *__restrict__ w, int64_t rows, int K,
                                      uint8_t *__restrict__ codes, uint8_t *__restrict__ scales) {
    const int64_t nb = K / 32;
    const int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (blk >= rows * nb) return;
    const int64_t r = blk / nb, b = blk % nb;
    const float4 *src = reinterpret_cast<const float4 *>(w + r * K + b * 32);
    float v[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float4 q = src[i];
        v[4 * i] = q.x; v[4 * i + 1] = q.y; v[4 * i + 2] = q.z; v[4 * i + 3] = q.w;
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    uint32_t packed[4] = {0, 0, 0, 0};
    uint8_t sb = 127;
    if (amax > 0.0f) {
        const int se = mx_shared_exp(amax, 2);
        sb = (uint8_t)(se + 127);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
            const uint32_t byte = f32x2_to_e2m1x2(ldexpf(v[i], -se), ldexpf(v[i + 1], -se));
            packed[i / 8] |= byte << (8 * ((i / 2) % 4));
        }
    }
    reinterpret_cast<uint4 *>(codes + r * (K / 2) + b * 16)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    scales[r * nb + b] = sb;
}

// One thread per Q2_K super-block (256 weights), the min-max rule in fp32:
// mn = max(0, -min w), rng = (max w + mn) / 3 per 16-sub-block; d = f16(max rng
// / 15), dmin = f16(max mn / 15); sc, m = round(rng / d), round(mn / dmin) in
// [0, 15]; q = round((w + dmin m) / (d sc)) in [0, 3]; zero divisors give 0.
__global__ void quantize_q2k_kernel(const float *__restrict__ w, int64_t nsb, uint8_t *__restrict__ out) {
    const int64_t sb = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (sb >= nsb) return;
    const float *v = w + sb * 256;
    uint8_t *o = out + sb * 84;
    float rng[16], mn[16], rmax = 0.0f, mmax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float lo = v[16 * i], hi = v[16 * i];
        for (int j = 1; j < 16; ++j) {
            lo = fminf(lo, v[16 * i + j]);
            hi = fmaxf(hi, v[16 * i + j]);
        }
        mn[i] = fmaxf(0.0f, -lo);
        rng[i] = __fdiv_rn(__fadd_rn(hi, mn[i]), 3.0f);
        rmax = fmaxf(rmax, rng[i]);
        mmax = fmaxf(mmax, mn[i]);
    }
    const __half dh = __float2half_rn(__fdiv_rn(rmax, 15.0f));
    const __half mh = __float2half_rn(__fdiv_rn(mmax, 15.0f));
    const float d = __half2float(dh), dmin = __half2float(mh);
    uint8_t qs[64];
    for (int i = 0; i < 64; ++i) qs[i] = 0;
    for (int i = 0; i < 16; ++i) {
        const int sc = d > 0.0f ? (int)fminf(fmaxf(roundf(__fdiv_rn(rng[i], d)), 0.0f), 15.0f) : 0;
        const int m = dmin > 0.0f ? (int)fminf(fmaxf(roundf(__fdiv_rn(mn[i], dmin)), 0.0f), 15.0f) : 0;
        o[i] = (uint8_t)(sc | (m << 4));
        for (int j = 0; j < 16; ++j) {
            const int n = 16 * i + j;
            int q = 0;
            if (sc > 0) {
                const float num = __fadd_rn(v[n], __fmul_rn(dmin, (float)m));
                q = (int)fminf(fmaxf(roundf(__fdiv_rn(num, __fmul_rn(d, (float)sc))), 0.0f), 3.0f);
            }
            qs[n / 4] |= (uint8_t)(q << (2 * (n % 4)));
        }
    }
    for (int i = 0; i < 64; ++i) o[16 + i] = qs[i];
    const uint16_t db = __half_as_ushort(dh), mb = __half_as_ushort(mh);
    o[80] = (uint8_t)(db & 0xFF);
    o[81] = (uint8_t)(db >> 8);
    o[82] = (uint8_t)(mb & 0xFF);
    o[83] = (uint8_t)(mb >> 8);
}

cudaError_t launch_quantize_weights(const moe_dims &d, int which, const float *w, uint8_t *canonical,
                                    cudaStream_t s) {
    int64_t N, K;
    mat_shape(d, which, N, K);
    const int64_t rows = (int64_t)d.E * N;
    if (d.wfmt == MOE_W_Q2K) {
        const int64_t nsb = rows * (K / 256);
        quantize_q2k_kernel<<<(unsigned)((nsb + 127) / 128), 128, 0, s>>>(w, nsb, canonical);
    } else {
        const int64_t nb = rows * (K / 32);
        quantize_mxfp4_kernel<<<(unsigned)((nb + 255) / 256), 256, 0, s>>>(w, rows, (int)K, canonical,
                                                                           canonical + rows * K / 2);
    }
    count_launches(1);
    return cudaGetLastError();
}

// Scale bytes, row-major [E*N][K/32] -> tiled atoms (see Mxfp4Layout).
__global__ void tile_scales_kernel(const uint8_t *__restrict__ srow, int64_t E, int64_t N, int64_t K,
                                   uint8_t *__restrict__ stile) {
    const int64_t nb = K / 32;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= E * N * nb) return;
    const int64_t kb = i % nb, n = (i / nb) % N, e = i / (nb * N);
    stile[mxfp4_tile_index(e, n, kb, N, K)] = srow[i];
}

// Q2_K super-blocks (84 bytes) -> split quants / scale bytes / (d, dmin).
__global__ void pack_q2k_kernel(const uint8_t *__restrict__ in, int64_t nsb, uint8_t *__restrict__ qs,
                                uint8_t *__restrict__ scm, uint32_t *__restrict__ dd) {
    const int64_t sb = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (sb >= nsb) return;
    const uint8_t *b = in + sb * 84;
    for (int i = 0; i < 16; ++i) scm[sb * 16 + i] = b[i];
    uint32_t words[16] = {};
    for (int e = 0; e < 256; ++e) {  // canonical: quant e at byte e / 4, bits 2 (e % 4)
        const uint32_t q = (b[16 + e / 4] >> (2 * (e % 4))) & 3u;
        words[q2k_word(e)] |= q << q2k_bit(e);
    }
    uint32_t *qw = reinterpret_cast<uint32_t *>(qs + sb * 64);
    for (int i = 0; i < 16; ++i) qw[i] = words[i];
    dd[sb] = (uint32_t)b[80] | (uint32_t)b[81] << 8 | (uint32_t)b[82] << 16 | (uint32_t)b[83] << 24;
}

cudaError_t launch_pack_weights(const moe_dims &d, int which, const uint8_t *canonical, uint8_t *packed,
                                cudaStream_t s) {
    if (d.wfmt == MOE_W_Q2K) {
        const Q2kLayout L = q2k_layout(d, which);
        const int64_t nsb = L.E * L.N * (L.K / 256);
        pack_q2k_kernel<<<(unsigned)((nsb + 255) / 256), 256, 0, s>>>(
            canonical, nsb, packed + L.qs, packed + L.scm, reinterpret_cast<uint32_t *>(packed + L.dd));
        count_launches(1);
        return cudaGetLastError();
    }
    const Mxfp4Layout L = mxfp4_layout(d, which);
    const int64_t ncode = L.E * L.N * L.K / 2, nsc = L.E * L.N * L.K / 32;
    cudaError_t err = cudaMemcpyAsync(packed + L.codes, canonical, ncode, cudaMemcpyDeviceToDevice, s);
    if (err != cudaSuccess) return err;
    err = cudaMemcpyAsync(packed + L.srow, canonical + ncode, nsc, cudaMemcpyDeviceToDevice, s);
    if (err != cudaSuccess) return err;
    tile_scales_kernel<<<(unsigned)((nsc + 255) / 256), 256, 0, s>>>(canonical + ncode, L.E, L.N, L.K,
                                                                     packed + L.stile);
    count_launches(1);
    return cudaGetLastError();
}

// Packed matrix of one expert -> fp32 [N][K]; exact decode.
__global__ void debug_dequant_kernel(const uint8_t *__restrict__ packed, int wfmt, int64_t E, int64_t N,
                                     int64_t K, int64_t off_a, int64_t off_b, int64_t off_c, int expert,
                                     float *__restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= N * K) return;
    const int64_t n = i / K, kk = i % K, row = (int64_t)expert * N + n;
    if (wfmt == MOE_W_Q2K) {
        const int64_t sb = row * (K / 256) + kk / 256, j = kk % 256;
        const uint8_t scm = packed[off_b + sb * 16 + j / 16];
        const uint32_t dd = reinterpret_cast<const uint32_t *>(packed + off_c)[sb];
        const float dv = __half2float(__ushort_as_half((uint16_t)(dd & 0xFFFF)));
        const float mv = __half2float(__ushort_as_half((uint16_t)(dd >> 16)));
        const uint32_t w = reinterpret_cast<const uint32_t *>(packed + off_a)[sb * 16 + q2k_word((int)j)];
        const int q = (int)((w >> q2k_bit((int)j)) & 3u);
        const float a = __fmul_rn(__fmul_rn(dv, (float)(scm & 15)), (float)q);
        out[i] = __fsub_rn(a, __fmul_rn(mv, (float)(scm >> 4)));
    } else {
        const uint8_t byte = packed[off_a + row * (K / 2) + kk / 2];
        const uint32_t code = (kk & 1) ? (byte >> 4) : (byte & 15);
        out[i] = e2m1_to_f32(code) * e8m0_to_f32(packed[off_b + row * (K / 32) + kk / 32]);
    }
}

cudaError_t launch_debug_dequant(const moe_dims &d, int which, const uint8_t *packed, int expert,
                                 float *out, cudaStream_t s) {
    int64_t N, K, a, b, c;
    if (d.wfmt == MOE_W_Q2K) {
        const Q2kLayout L = q2k_layout(d, which);
        N = L.N; K = L.K; a = L.qs; b = L.scm; c = L.dd;
    } else {
        const Mxfp4Layout L = mxfp4_layout(d, which);
        N = L.N; K = L.K; a = L.codes; b = L.srow; c = 0;
    }
    const int64_t n = N * K;
    debug_dequant_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(packed, d.wfmt, d.E, N, K, a, b, c,
                                                                     expert, out);
    count_launches(1);
    return cudaGetLastError();
}

// MXFP8 (E4M3 elements): one thread per 32-block; the power-of-two scaling is
// exact, so the codes depend only on the inputs, never on evaluation order.
template <typename T>
__device__ __forceinline__ float load_act(const T *p, int64_t i);
template <>
__device__ __forceinline__ float load_act<uint16_t>(const uint16_t *p, int64_t i) { return bf16_to_f32(p[i]); }
template <>
__device__ __forceinline__ float load_act<float>(const float *p, int64_t i) { return p[i]; }

// One thread per 32-element block: MXFP8 (AF 8, E4M3 codes [rows][K]) or
// MXFP4 (AF 4, E2M1 codes [rows][K/2], element 2i in the low nibble), E8M0
// scales [rows][K/32]; the OCP rule with emax 8 or 2.
template <typename T, int AF>
__global__ void quant_act_kernel(const T *__restrict__ x, int64_t rows, int K, uint8_t *__restrict__ codes,
                                 uint8_t *__restrict__ scales) {
    const int64_t nb = K / 32;
    const int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (blk >= rows * nb) return;
    const int64_t base = (blk / nb) * K + (blk % nb) * 32;
    float v[32], amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        v[i] = load_act<T>(x, base + i);
        amax = fmaxf(amax, fabsf(v[i]));
    }
    uint32_t packed[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    uint8_t sb = 127;
    if (amax > 0.0f) {
        const int se = mx_shared_exp(amax, AF == 8 ? 8 : 2);
        sb = (uint8_t)(se + 127);
#pragma unroll
        for (int i = 0; i < 32; i += AF == 8 ? 1 : 2) {
            if (AF == 8) {
                const uint32_t c = __nv_cvt_float_to_fp8(ldexpf(v[i], -se), __NV_SATFINITE, __NV_E4M3);
                packed[i / 4] |= c << (8 * (i % 4));
            } else {
                packed[i / 8] |= f32x2_to_e2m1x2(ldexpf(v[i], -se), ldexpf(v[i + 1], -se)) << (8 * ((i / 2) % 4));
            }
        }
    }
    if (AF == 8) {
        uint4 *dst = reinterpret_cast<uint4 *>(codes + base);
        dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    } else {
        *reinterpret_cast<uint4 *>(codes + base / 2) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
    scales[blk] = sb;
}

cudaError_t launch_quant_act_bf16(const uint16_t *x, int64_t rows, int K, uint8_t *codes, uint8_t *scales,
                                  cudaStream_t s, bool fp4) {
    const int64_t nb = rows * (K / 32);
    if (nb == 0) return cudaSuccess;
    const unsigned g = (unsigned)((nb + 255) / 256);
    if (fp4) quant_act_kernel<uint16_t, 4><<<g, 256, 0, s>>>(x, rows, K, codes, scales);
    else quant_act_kernel<uint16_t, 8><<<g, 256, 0, s>>>(x, rows, K, codes, scales);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_quant_act_f32(const float *x, int64_t rows, int K, uint8_t *codes, uint8_t *scales,
                                 cudaStream_t s, bool fp4) {
    const int64_t nb = rows * (K / 32);
    if (nb == 0) return cudaSuccess;
    const unsigned g = (unsigned)((nb + 255) / 256);
    if (fp4) quant_act_kernel<float, 4><<<g, 256, 0, s>>>(x, rows, K, codes, scales);
    else quant_act_kernel<float, 8><<<g, 256, 0, s>>>(x, rows, K, codes, scales);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
