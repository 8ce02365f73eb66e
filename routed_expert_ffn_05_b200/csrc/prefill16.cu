// Batched expert FFN with bf16 activations ("w4a16") on the 5th-generation
// tensor cores, for the batches the decode kernel does not take (T > 8, or
// other dims).
//
// The routed experts are MXFP4 and their batched work belongs on the tensor
// cores ("DwarfStar", hysenlabs.com, "Model support and quantisation"); here
// the activations stay bf16, so the MMA is kind::f16 with bf16 operands and
// the weights are decoded on the fly: E2M1 x 2^(e - 127) is exact in bf16
// (at most two significant bits, the fp32 exponent range), so the products are
// exact and only the fp32 accumulation rounds.
//
// Mapping onto tcgen05.mma (kind::f16, K = 16 per instruction):
//  - A = 128 weight rows, decoded into TENSOR memory by four decoder warps
//    (thread = weight row = TMEM lane: 64 codes and two scales per stage become
//    32 bf16 pairs, one tcgen05.st of 32 columns), so the decoded tile never
//    passes through shared memory; the packed codes arrive by TMA (32 bytes
//    per row and stage) in the same shared-memory stage as the token rows,
//    with the tile's E8M0 scale atom (128 rows x K 128, the layout the
//    block-scaled path reads) beside them;
//  - B = a tile of 128 of the expert's token rows (bf16, K-major, 128-byte
//    swizzled TMA boxes of K = 64); gate/up: the gathered x rows, down: h;
//  - gate/up runs two MMAs per K step into two accumulators (g from W1 rows,
//    u from the same W3 rows), down one;
//  - the epilogue thread is a weight row (TMEM lane), its columns tokens:
//    h = bf16(silu(g) u) goes to h [S][d_ff] (K-major for the down GEMM), the
//    down rows to out_rows [S][d_model] in fp32.
// One persistent CTA per SM: a TMA warp, an MMA warp, four decoder warps and
// eight epilogue warps; an 8-stage shared-memory ring (token rows + codes)
// ahead of a 4-stage tensor-memory ring (decoded A); every wait is bounded.
#include <string.h>

#include <atomic>

#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tma.h"

namespace moe {
namespace {

constexpr int k16Sm = 8;          // shared-memory stages: token rows and weight codes
constexpr int k16Ta = 4;          // tensor-memory stages: decoded weights
constexpr int k16Dec = 1;         // decoder warps per TMEM lane quarter (they would take turns by stage;
                                  // three measured 5% slower: the MMAs, not the decoders, set the pace)
constexpr int k16Epi = 2;         // epilogue warps per TMEM lane quarter (each a share of the tokens)
constexpr int k16Threads = 32 * (2 + 4 * k16Dec + 4 * k16Epi);  // warp 0 TMA, 1 MMA, decoders, epilogue
constexpr int k16Tile = 128;      // weight rows (M) and tokens (N) per tile
constexpr int k16Kst = 64;        // K per stage (one 128-byte row of bf16)
constexpr int k16MaxE = 1024;
constexpr uint32_t k16Cols = 512;

enum { kGU16 = 0, kDN16 = 1 };

struct T16Args {
    CUtensorMap act;              // token rows bf16 [S][K], 64 x 128 boxes, 128-byte swizzled
    CUtensorMap wcm[2];           // packed E2M1 codes [E * Nw][K / 2], 32-byte x 128-row boxes, 32-byte
                                  // swizzled: gate/up W1, W3; down W2
    const uint8_t *wsf[2];        // E8M0 scale atoms [E][Nw / 128][K / 128][512] (layout.h)
    const int32_t *offsets, *ustart;
    int E, Nw, K;                 // weight rows per expert, input dim
    uint16_t *h;                  // gate/up: h bf16 [S][Nw]
    float *out;                   // down: rows fp32 [S][Nw]
    int *err;
};

struct T16Smem {
    uint8_t b[k16Sm][k16Tile * 128];      // token rows: 128 rows x K 64 (bf16)
    uint8_t wc[k16Sm][2][k16Tile * 32];   // weight codes: 128 rows x K 64 (E2M1) per matrix
    uint8_t wsf[k16Sm][2][512];           // the scale atom holding the stage's K 64 per matrix
    uint64_t full[k16Sm], sempty[k16Sm], a_full[k16Ta], aempty[k16Ta], acc_full[2], acc_empty[2], mma_done;
    uint32_t tmem_base;
    volatile int abort;
    int ustart[k16MaxE + 1];
};
constexpr int k16SmemBytes = (int)sizeof(T16Smem) + 1024;

__device__ __forceinline__ T16Smem &t16_smem(uint8_t *raw) {
    return *reinterpret_cast<T16Smem *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
}

struct Work16 {
    int e, f, j, row0, nvalid;
};

// Work item w -> (expert, 128-row weight tile, token tile), weight-tile-major
// within an expert (CTAs on neighbouring items share the weight tile in L2).
__device__ __forceinline__ Work16 work16_of(int w, int ft, const int *ustart, int E, const int32_t *offsets) {
    const int v = w / ft;
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (ustart[mid] <= v) lo = mid;
        else hi = mid - 1;
    }
    const int e = lo, nt = ustart[e + 1] - ustart[e], local = w - ft * ustart[e];
    Work16 wk;
    wk.e = e;
    wk.f = local / nt;
    wk.j = local % nt;
    wk.row0 = offsets[e] + k16Tile * wk.j;
    wk.nvalid = min(k16Tile, offsets[e + 1] - wk.row0);
    return wk;
}

__device__ __forceinline__ void t16_fail(const T16Args &a, T16Smem &s) {
    set_device_error(a.err, MOE_DEVERR_TIMEOUT);
    s.abort = 1;
}

// Two fp32 -> bf16x2 (round to nearest even; exact for the decoded weights).
__device__ __forceinline__ uint32_t f32x2_to_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// (lo, hi) * (s, s) as one packed fp32 multiply, round to nearest even.
__device__ __forceinline__ float2 mul_f32x2(float2 v, float sc) {
    uint64_t p, q, r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(p) : "f"(v.x), "f"(v.y));
    asm("mov.b64 %0, {%1, %1};" : "=l"(q) : "f"(sc));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(p), "l"(q));
    float2 o;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(o.x), "=f"(o.y) : "l"(r));
    return o;
}

// 64 E2M1 codes (32 bytes, element 2i in the low nibble of byte i) of one
// weight row and their two E8M0 scales -> 32 bf16 pairs, element order.
__device__ __forceinline__ void decode64(const uint4 c[2], uint32_t sc2, uint32_t (&o)[32]) {
    const float s0 = e8m0_to_f32(sc2 & 0xFFu), s1 = e8m0_to_f32((sc2 >> 8) & 0xFFu);
    const uint32_t w[8] = {c[0].x, c[0].y, c[0].z, c[0].w, c[1].x, c[1].y, c[1].z, c[1].w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint32_t hh[4];
        e2m1x8_to_f16x8(w[i], hh);  // byte b of w -> hh[b] = (element 2b, 2b + 1) of the word's 8
        const float sc = i < 4 ? s0 : s1;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const __half2 h2 = *reinterpret_cast<const __half2 *>(&hh[b]);
            const float2 f = mul_f32x2(__half22float2(h2), sc);
            o[4 * i + b] = f32x2_to_bf16x2(f.x, f.y);
        }
    }
}

template <int MODE>
__global__ void __launch_bounds__(k16Threads, 1) tc16_ffn_kernel(const __grid_constant__ T16Args a) {
    extern __shared__ uint8_t smem_raw[];
    T16Smem &s = t16_smem(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool GU = MODE == kGU16;
    constexpr int kMats = GU ? 2 : 1;          // weight matrices per item: W1 and W3, or W2
    // accumulator columns: gate/up one buffer of g | u (256); down two buffers
    // of o (128 each), so the epilogue of one item overlaps the next item's MMAs
    constexpr int kNb = GU ? 1 : 2;
    constexpr uint32_t kAcc = 256u;              // A stages start here
    constexpr uint32_t kAStage = 32u * kMats;    // A columns per stage
    const int ft = a.Nw / k16Tile, kt_n = a.K / k16Kst;

    if (threadIdx.x == 0) {
        for (int i = 0; i < k16Sm; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.sempty[i], 1);
        }
        for (int i = 0; i < k16Ta; ++i) {
            mbar_init(&s.a_full[i], 4);  // one arrival per decoder warp
            mbar_init(&s.aempty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.acc_full[i], 1);
            mbar_init(&s.acc_empty[i], 4 * k16Epi);
        }
        mbar_init(&s.mma_done, 1);
        s.abort = 0;
        fence_mbar_init();
    }
    for (int i = threadIdx.x; i <= a.E; i += blockDim.x) s.ustart[i] = a.ustart[i];
    if (warp == 1) {
        tmem_alloc(&s.tmem_base, k16Cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;
    const int n_work = ft * s.ustart[a.E];

    if (warp == 0) {
        // ---------------------- TMA: token rows and weight codes ----------------------
        if (lane == 0) {
            prefetch_tensormap(&a.act);
            prefetch_tensormap(&a.wcm[0]);
            if (GU) prefetch_tensormap(&a.wcm[1]);
            int it = 0;
            for (int w = blockIdx.x; w < n_work && !s.abort; w += gridDim.x) {
                const Work16 wk = work16_of(w, ft, s.ustart, a.E, a.offsets);
                const int wrow = wk.e * a.Nw + wk.f * k16Tile;
                for (int kt = 0; kt < kt_n; ++kt, ++it) {
                    const int slot = it % k16Sm;
                    if (!mbar_wait(&s.sempty[slot], ((it / k16Sm) & 1) ^ 1, &s.abort)) { t16_fail(a, s); break; }
                    mbar_arrive_expect_tx(&s.full[slot], k16Tile * 128 + kMats * (k16Tile * 32 + 512));
                    tma_load_2d(s.b[slot], &a.act, kt * 128, wk.row0, &s.full[slot]);
                    const int64_t atom = ((int64_t)wrow / k16Tile) * (a.K / 128) + (kt >> 1);
#pragma unroll
                    for (int m = 0; m < kMats; ++m) {
                        tma_load_2d(s.wc[slot][m], &a.wcm[m], kt * 32, wrow, &s.full[slot]);
                        bulk_g2s(s.wsf[slot][m], a.wsf[m] + atom * 512, 512, &s.full[slot]);
                    }
                }
            }
            for (int g = it - k16Sm; g < it; ++g)  // copies in flight land before the CTA exits
                if (g >= 0) mbar_wait(&s.full[g % k16Sm], (g / k16Sm) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(k16Tile, k16Tile);
            int it = 0, lw = 0;
            for (int w = blockIdx.x; w < n_work && !s.abort; w += gridDim.x, ++lw) {
                const int ab = lw % kNb;  // accumulator buffer of this item
                if (!mbar_wait(&s.acc_empty[ab], ((lw / kNb) & 1) ^ 1, &s.abort)) { t16_fail(a, s); break; }
                tc_fence_after();
                const uint32_t dacc = tmem + 128u * (uint32_t)ab;
                bool ok = true;
                for (int kt = 0; kt < kt_n; ++kt, ++it) {
                    const int slot = it % k16Sm, ta = it % k16Ta;
                    if (!mbar_wait(&s.full[slot], (it / k16Sm) & 1, &s.abort) ||
                        !mbar_wait(&s.a_full[ta], (it / k16Ta) & 1, &s.abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t db = sdesc_sw128(s.b[slot]);
                    const uint32_t a0 = tmem + kAcc + kAStage * ta;
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {  // K = 16: 8 TMEM columns of A, 32 bytes of every B row
                        const uint32_t acc = (kt | ks) != 0;
                        tc_mma_bf16_ts(dacc, a0 + 8 * ks, db + 2 * ks, idesc, acc);
                        if (GU) tc_mma_bf16_ts(tmem + 128, a0 + 32 + 8 * ks, db + 2 * ks, idesc, acc);
                    }
                    tc_commit(&s.sempty[slot]);  // the shared stage and
                    tc_commit(&s.aempty[ta]);    // the A columns are free once these finish
                }
                if (!ok) { t16_fail(a, s); break; }
                tc_commit(&s.acc_full[ab]);
            }
            tc_commit(&s.mma_done);
            mbar_wait(&s.mma_done, 0);
        }
    } else if (warp < 2 + 4 * k16Dec) {
        // ------------------------------ decoders ------------------------------
        // thread = weight row r of the item's tile = TMEM lane r (this warp's
        // lane quarter q); the warp decodes the stages with it % k16Dec == j:
        // per stage the row's 32 code bytes of each matrix from the shared
        // stage (32-byte swizzle: half c of row r at c ^ (r / 4 % 2)) and its
        // four scale bytes of the atom (32-blocks 4 (kt / 2) .. + 3)
        const int q = warp & 3, j = (warp - 2) >> 2, r = 32 * q + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        const int h0 = 16 * ((r >> 2) & 1), h1 = 16 - h0;  // byte offsets of the row's halves 0, 1
        const int sfo = (r & 31) * 16 + (r >> 5) * 4;       // the row's scale word in an atom
        int it = 0;
        for (int w = blockIdx.x; w < n_work; w += gridDim.x) {
            if (__shfl_sync(0xffffffffu, s.abort, 0)) break;
            bool ok = true;
            for (int kt = 0; kt < kt_n; ++kt, ++it) {
                if (it % k16Dec != j) continue;
                const int slot = it % k16Sm, ta = it % k16Ta;
                ok = mbar_wait(&s.full[slot], (it / k16Sm) & 1, &s.abort) &&
                     mbar_wait(&s.aempty[ta], ((it / k16Ta) & 1) ^ 1, &s.abort);
                if (!__all_sync(0xffffffffu, ok)) break;
                tc_fence_after();
#pragma unroll
                for (int m = 0; m < kMats; ++m) {
                    const uint8_t *row = s.wc[slot][m] + 32 * r;
                    const uint4 c[2] = {lds128(row + h0), lds128(row + h1)};
                    const uint32_t sw = lds32(s.wsf[slot][m] + sfo) >> (16 * (kt & 1));  // bytes 2 (kt % 2), + 1
                    uint32_t o[32];
                    decode64(c, sw, o);
                    tmem_st32(lane_base + kAcc + kAStage * ta + 32 * m, o);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.a_full[ta]);
            }
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) t16_fail(a, s);
                break;
            }
        }
    } else {
        // ------------------------------ epilogue ------------------------------
        // TMEM lane = weight row (this warp: quarter q), columns = the tile's
        // tokens in chunks of 32; epilogue warp e of a quarter takes chunks
        // e, e + k16Epi, ...
        const int q = warp & 3, e = (warp - 2 - 4 * k16Dec) >> 2, r = 32 * q + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        int lw = 0;
        for (int w = blockIdx.x; w < n_work; w += gridDim.x, ++lw) {
            if (__shfl_sync(0xffffffffu, s.abort, 0)) break;
            const Work16 wk = work16_of(w, ft, s.ustart, a.E, a.offsets);
            const int ab = lw % kNb;
            const bool ok = mbar_wait(&s.acc_full[ab], (lw / kNb) & 1, &s.abort);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) t16_fail(a, s);
                break;
            }
            tc_fence_after();
            const int col = wk.f * k16Tile + r;  // this thread's output feature (gate/up: row of h)
            // the accumulator goes back as soon as this warp's last chunk is in registers
            int last = -1;
            for (int cc = e; cc < 4; cc += k16Epi)
                if (32 * cc < wk.nvalid) last = cc;
            auto release = [&]() {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.acc_empty[ab]);
            };
            if (last < 0) release();
#pragma unroll 1
            for (int cc = e; cc <= last; cc += k16Epi) {
                const int t0 = 32 * cc;            // first token of this chunk
                uint32_t g[32], u[32];
                tmem_ld32(lane_base + 128u * (uint32_t)ab + t0, g);
                if (GU) tmem_ld32(lane_base + 128 + t0, u);
                tmem_wait_ld();
                if (cc == last) release();
                const int nv = min(32, wk.nvalid - t0);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if (i >= nv) break;
                    const int64_t o = (int64_t)(wk.row0 + t0 + i) * a.Nw + col;
                    if (GU) a.h[o] = f32_to_bf16_rne(silu_f32(__uint_as_float(g[i])) * __uint_as_float(u[i]));
                    else a.out[o] = __uint_as_float(g[i]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, k16Cols);
    }
}

// One warp per token: its bf16 x row to each of its k rows (expert order).
__global__ void __launch_bounds__(256) tc16_gather_kernel(const uint16_t *__restrict__ x,
                                                          const int32_t *__restrict__ row_of, int T, int k, int d,
                                                          uint16_t *__restrict__ gx) {
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (t >= T) return;
    int rows[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) rows[j] = j < k ? __ldg(&row_of[(int64_t)t * k + j]) : -1;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (int64_t)t * d);
    for (int i = lane; i < d / 8; i += 32) {
        const uint4 v = __ldg(src + i);
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (j < k && rows[j] >= 0) reinterpret_cast<uint4 *>(gx + (int64_t)rows[j] * d)[i] = v;
    }
}

int tc16_num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

cudaError_t tc16_set_attrs() {
    static std::atomic<bool> done[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(tc16_ffn_kernel<kGU16>, cudaFuncAttributeMaxDynamicSharedMemorySize, k16SmemBytes)))
        return e;
    if ((e = cudaFuncSetAttribute(tc16_ffn_kernel<kDN16>, cudaFuncAttributeMaxDynamicSharedMemorySize, k16SmemBytes)))
        return e;
    done[dev].store(true, std::memory_order_release);
    return cudaSuccess;
}

}  // namespace

bool tc16_path_applies(const moe_dims &d) {
    return d.wfmt == MOE_W_MXFP4 && d.act == MOE_A_BF16 && !decode_path_applies(d) && d.T >= 1 &&
           d.d_model % k16Tile == 0 && d.d_ff % k16Tile == 0 && d.E <= k16MaxE;
}

// Routed expert FFN, bf16 activations and MXFP4 weights, on the tensor cores:
// plan, gather of the bf16 rows in expert order, gate/up GEMM with SwiGLU
// (h rounded to bf16), down GEMM into fp32 rows.
cudaError_t launch_tc16_ffn(const moe_dims &d, const moe_weights &w, const uint16_t *x, const int32_t *offsets,
                            const int32_t *perm, float *out_rows, uint8_t *ws, const WsLayout &L, cudaStream_t s) {
    const int S = d.T * d.k;
    if (S == 0) return cudaSuccess;
    cudaError_t e = tc16_set_attrs();
    if (e != cudaSuccess) return e;
    const Mxfp4Layout L1 = mxfp4_layout(d, MOE_MAT_W1), L2 = mxfp4_layout(d, MOE_MAT_W2);
    const uint8_t *p1 = static_cast<const uint8_t *>(w.w1), *p3 = static_cast<const uint8_t *>(w.w3),
                  *p2 = static_cast<const uint8_t *>(w.w2);
    int32_t *ustart = reinterpret_cast<int32_t *>(ws + L.ustart);
    int32_t *row_of = reinterpret_cast<int32_t *>(ws + L.row_of);
    uint16_t *h = reinterpret_cast<uint16_t *>(ws + L.h);  // [S][F] bf16 (the region is sized for fp32)
    // the gathered x rows [S][d] bf16 are staged in out_rows ([S][d] fp32, twice their size): the
    // gate/up GEMM reads them before the down GEMM, later in stream order, writes the rows
    uint16_t *gx = reinterpret_cast<uint16_t *>(out_rows);
    T16Args g, dn;
    memset(&g, 0, sizeof g);
    memset(&dn, 0, sizeof dn);
    const uint64_t r13 = (uint64_t)d.E * d.d_ff, r2 = (uint64_t)d.E * d.d_model;
    if (!make_tile_map_u8(&g.act, gx, S, (uint64_t)d.d_model * 2, k16Tile) ||
        !make_tile_map_u8(&dn.act, h, S, (uint64_t)d.d_ff * 2, k16Tile) ||
        !make_rows32_map(&g.wcm[0], p1 + L1.codes, r13, (uint64_t)d.d_model / 2, k16Tile) ||
        !make_rows32_map(&g.wcm[1], p3 + L1.codes, r13, (uint64_t)d.d_model / 2, k16Tile) ||
        !make_rows32_map(&dn.wcm[0], p2 + L2.codes, r2, (uint64_t)d.d_ff / 2, k16Tile))
        return cudaErrorInvalidValue;
    g.wsf[0] = p1 + L1.stile; g.wsf[1] = p3 + L1.stile;
    g.offsets = offsets; g.ustart = ustart; g.E = d.E; g.Nw = d.d_ff; g.K = d.d_model; g.h = h;
    g.err = device_error_word();
    dn.wsf[0] = p2 + L2.stile;
    dn.offsets = offsets; dn.ustart = ustart; dn.E = d.E; dn.Nw = d.d_model; dn.K = d.d_ff; dn.out = out_rows;
    dn.err = g.err;
    if ((e = launch_tc_plan(d, offsets, perm, ustart, row_of, s)) != cudaSuccess) return e;
    tc16_gather_kernel<<<(d.T + 7) / 8, 256, 0, s>>>(x, row_of, d.T, d.k, d.d_model, gx);
    const int grid = tc16_num_sms();
    tc16_ffn_kernel<kGU16><<<grid, k16Threads, k16SmemBytes, s>>>(g);
    tc16_ffn_kernel<kDN16><<<grid, k16Threads, k16SmemBytes, s>>>(dn);
    count_launches(3);
    return cudaGetLastError();
}

}  // namespace moe
