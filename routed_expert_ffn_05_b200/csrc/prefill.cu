// Prefill-sized expert FFN in w4a8 mode on the 5th-generation tensor cores:
// block-scaled MMA of E2M1 weights against E4M3 activations, both with E8M0
// scales per 32 along K (OCP MX v1.0), fp32 accumulate in tensor memory.
//
// The routed experts are FP4 and the expert work is batched per expert ("DS4",
// dibi8.com, "Key architectural innovations" item 1; "DwarfStar",
// hysenlabs.com, "Model support and quantisation"). The layer's math:
// g = W1 a, u = W3 a, h = silu(g) * u quantised to MXFP8 along F, o = W2 h.
//
// Mapping onto tcgen05.mma (K = 32 per instruction):
//  - A is a tile of 128 of the expert's tokens (M = 128, E4M3) and B is 256
//    weight rows (N = 256, E2M1): for gate/up the 128 rows of W1 and the same
//    128 rows of W3 stacked, for down 256 rows of W2. One MMA per K step then
//    gives g and u (or 256 output features) for every token of the tile. An
//    instruction costs the same at N = 128 as at N = 64 or 32 (its 128 x 32
//    A read sets the time), and N = 256 costs ~1.1x N = 128, so one 256-wide
//    MMA does the work of two 128-wide ones in ~55% of their time;
//    token tiles that are not full (the routing is skewed, many experts get a
//    few tokens) cost a full tile either way;
//  - the epilogue thread is a token (a TMEM lane): SwiGLU pairs columns c and
//    128 + c, the MXFP8 amax of h along F is 32 values of the same thread, and
//    h codes and output rows leave as contiguous 16-byte stores;
//  - operands arrive by TMA in 128-byte-swizzled K-major boxes of 128 K; E2M1
//    codes are expanded to one byte per element in shared memory by the
//    tensor map's 16U4_ALIGN16B type; the E8M0 scales come in 512-byte atoms
//    (128 rows x 4 blocks) that tcgen05.cp broadcasts into tensor memory;
//  - one persistent CTA per SM: a TMA warp, an MMA warp and eight epilogue
//    warps, a 4-stage mbarrier ring; every wait is bounded.
#include <string.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tma.h"

namespace moe {
namespace {

constexpr int kTcStages = 4;
constexpr int kTcThreads = 320;   // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr int kTileBytes = 16384; // 128 rows x 128 bytes
constexpr uint32_t kTmemCols = 512;
constexpr int kSfCol = 256;       // scale-factor columns: 16 per stage from here
constexpr int kTcMaxE = 1024;
constexpr int kTile = 128;        // weight rows and tokens per tile, K per stage

enum { kModeGU = 0, kModeDN = 1 };

struct TcArgs {
    CUtensorMap wa, wb;  // weights: W1 and W3 (gate/up) or W2 (down), E2M1 expanded
    CUtensorMap act;     // activations: gathered x codes (gate/up) or h codes (down)
    const uint8_t *sfa, *sfb;  // weight scale atoms (W1/W2, W3)
    const uint8_t *sfact;      // activation scale atoms per token tile
    const int32_t *offsets;    // [E+1] expert row ranges
    const int32_t *ustart;     // [E+1] token-tile prefix
    int E, Nw, K;              // weight rows per expert, K
    uint8_t *h8;               // gate/up: h codes [S][F]
    uint8_t *hsf;              // gate/up: h scale atoms [tiles][F/128][512]
    float *out;                // down: rows [S][d] fp32, or
    uint16_t *out16;           //       bf16 when this is set
    int *err;
};

struct TcSmem {
    uint8_t a[kTcStages][2][kTileBytes];
    uint8_t b[kTcStages][kTileBytes];
    uint8_t sf[kTcStages][3][1024];  // E8M0 atoms per stage: W (rows 0..127), W (128..255), tokens
    uint64_t full[kTcStages], empty[kTcStages], acc_full, acc_empty, mma_done;
    uint32_t tmem_base;
    volatile int abort;
    int ustart[kTcMaxE + 1];
};
constexpr int kTcSmemBytes = (int)sizeof(TcSmem) + 1024;

__device__ __forceinline__ TcSmem &tc_smem(uint8_t *raw) {
    return *reinterpret_cast<TcSmem *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
}

struct Work {
    int e, f, j, row0, nvalid;
};

// Work item w -> (expert, weight tile, token tile). Items of one expert are
// ordered weight-tile-major, so CTAs running neighbouring items share the same
// weight tile through L2.
__device__ __forceinline__ Work work_of(int w, int ft, const int *ustart, int E, const int32_t *offsets) {
    const int v = w / ft;
    int lo = 0, hi = E - 1;  // largest e with ustart[e] <= v
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (ustart[mid] <= v) lo = mid;
        else hi = mid - 1;
    }
    const int e = lo, nt = ustart[e + 1] - ustart[e];
    const int local = w - ft * ustart[e];
    Work wk;
    wk.e = e;
    wk.f = local / nt;
    wk.j = local % nt;
    wk.row0 = offsets[e] + kTile * wk.j;
    wk.nvalid = min(kTile, offsets[e + 1] - wk.row0);
    return wk;
}

__device__ __forceinline__ void tc_fail(const TcArgs &a, TcSmem &s) {
    set_device_error(a.err, MOE_DEVERR_TIMEOUT);
    s.abort = 1;
}

// Byte of the scale of (row t of a 128-row tile, 32-block q of a 128-wide K
// atom) inside the atom: the order tcgen05.cp 32x128b.warpx4 spreads over TMEM.
__device__ __forceinline__ int sf_atom_byte(int t, int q) { return (t & 31) * 16 + (t >> 5) * 4 + q; }

__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(r) : "f"(lo), "f"(hi));
    return r;
}

// Eight fp32 values times sc -> eight E2M1 codes in one word (element i in
// bits 4i .. 4i + 3), round to nearest even, saturating (hardware conversion).
__device__ __forceinline__ uint32_t e2m1x8(const float *v, float sc) {
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t b;
        asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
            : "=r"(b) : "f"(v[2 * i + 1] * sc), "f"(v[2 * i] * sc));
        w |= b << (8 * i);
    }
    return w;
}

// Two fp32 -> bf16 (round to nearest even), the first in the low half.
__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
    return (uint32_t)f32_to_bf16_rne(lo) | (uint32_t)f32_to_bf16_rne(hi) << 16;
}

// 2^-se as an fp32 (exact for se in [-127, 126]).
__device__ __forceinline__ float pow2_neg(int se) { return __uint_as_float((uint32_t)(127 - se) << 23); }

// AF: the activations' element bits. 8: E4M3 tokens against E2M1 weights on
// kind::mxf8f6f4 (the weights expanded to a byte per element by the tensor
// map; one 128-byte row of a box is K = 128, one MMA is K = 32). 4: E2M1 on
// both sides on kind::mxf4 (packed two per byte; a box row is K = 256, one
// MMA is K = 64 with two E8M0 scales per row, scale_vec::2X).
template <int MODE, int AF>
__global__ void __launch_bounds__(kTcThreads, 1) tc_ffn_kernel(const __grid_constant__ TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    TcSmem &s = tc_smem(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool GU = MODE == kModeGU;
    constexpr int kKs = AF == 8 ? kTile : 2 * kTile;   // K per stage
    constexpr int kAt = kKs / 128;                     // E8M0 atoms (128 rows x 128 K) per operand per stage
    constexpr int kSfStage = AF == 8 ? 16 : 24;        // TMEM scale columns per stage
    // work items per expert and token tile: 128 gate+up rows (gate/up) or 256
    // down rows (down), both as two 128-row MMA operands per K step
    const int ft = a.Nw / (GU ? kTile : 2 * kTile), kt_n = a.K / kKs, at_n = a.K / 128;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kTcStages; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1);
        }
        mbar_init(&s.acc_full, 1);
        mbar_init(&s.acc_empty, 8);
        mbar_init(&s.mma_done, 1);
        s.abort = 0;
        fence_mbar_init();
    }
    for (int i = threadIdx.x; i <= a.E; i += blockDim.x) s.ustart[i] = a.ustart[i];
    if (warp == 1) {
        tmem_alloc(&s.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;
    const int n_work = ft * s.ustart[a.E];

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            prefetch_tensormap(&a.wa);
            prefetch_tensormap(&a.act);
            // an expanded E2M1 box credits the packed bytes it reads (8 KB), not
            // the 16 KB it fills in shared memory; packed boxes credit 16 KB
            const uint32_t tx = (AF == 8 ? kTileBytes : 2 * kTileBytes) + kTileBytes + 3 * 512 * kAt;
            int it = 0;
            for (int w = blockIdx.x; w < n_work && !s.abort; w += gridDim.x) {
                const Work wk = work_of(w, ft, s.ustart, a.E, a.offsets);
                // the two weight tiles: W1 and W3 rows 128 f (gate/up), W2 rows 256 f and 256 f + 128 (down)
                const int wrow0 = wk.e * a.Nw + wk.f * (GU ? kTile : 2 * kTile), wrow1 = GU ? wrow0 : wrow0 + kTile;
                const int64_t rg0 = (int64_t)wk.e * (a.Nw / kTile) + (GU ? wk.f : 2 * wk.f);  // 128-row group
                const int64_t wat0 = rg0 * at_n, wat1 = (GU ? rg0 : rg0 + 1) * at_n;        // weight atom bases
                const int64_t aat = ((int64_t)s.ustart[wk.e] + wk.j) * at_n;              // activation atom base
                for (int kt = 0; kt < kt_n; ++kt, ++it) {
                    const int slot = it % kTcStages;
                    if (!mbar_wait(&s.empty[slot], ((it / kTcStages) & 1) ^ 1)) { tc_fail(a, s); break; }
                    uint64_t *bar = &s.full[slot];
                    mbar_arrive_expect_tx(bar, tx);
                    // box x coordinate: 128 K-elements (AF 8, expanded map) or 128 bytes = 256 K (AF 4)
                    tma_load_2d(s.a[slot][0], &a.wa, kt * kTile, wrow0, bar);
                    tma_load_2d(s.a[slot][1], &a.wb, kt * kTile, wrow1, bar);
                    tma_load_2d(s.b[slot], &a.act, kt * kTile, wk.row0, bar);
                    bulk_g2s(s.sf[slot][0], a.sfa + (wat0 + kAt * kt) * 512, 512 * kAt, bar);
                    bulk_g2s(s.sf[slot][1], a.sfb + (wat1 + kAt * kt) * 512, 512 * kAt, bar);
                    bulk_g2s(s.sf[slot][2], a.sfact + (aat + kAt * kt) * 512, 512 * kAt, bar);
                }
            }
            // copies in flight land before the CTA exits
            for (int g = it - kTcStages; g < it; ++g)
                if (g >= 0) mbar_wait(&s.full[g % kTcStages], (g / kTcStages) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            int it = 0, lw = 0;
            for (int w = blockIdx.x; w < n_work && !s.abort; w += gridDim.x, ++lw) {
                // A = the token tile (E4M3 or E2M1, M = 128), B = both 128-row
                // weight tiles as one 256-row operand (E2M1, N = 256): one MMA per
                // K step yields gate and up (or 256 down features) for every token
                // (format codes: mxf8f6f4 E4M3 0, E2M1 5; mxf4 E2M1 1)
                constexpr uint32_t idesc = AF == 8 ? idesc_mx(0, 5, 128, 256) : idesc_mx(1, 1, 128, 256);
                if (!mbar_wait(&s.acc_empty, (lw & 1) ^ 1)) { tc_fail(a, s); break; }
                tc_fence_after();
                bool ok = true;
                for (int kt = 0; kt < kt_n; ++kt, ++it) {
                    const int slot = it % kTcStages;
                    if (!mbar_wait(&s.full[slot], (it / kTcStages) & 1)) { ok = false; break; }
                    tc_fence_after();
                    // scale columns of atom at (K 128 at .. + 127): weight rows 0..127 at
                    // +8 at, 128..255 at +8 at + 4 (B reads column n / 32), tokens at
                    // +8 kAt + 4 at (A reads column m / 32); a column's byte j is 32-block j
                    const uint32_t sfc = tmem + kSfCol + kSfStage * slot;
#pragma unroll
                    for (int at = 0; at < kAt; ++at) {
                        tc_cp_sf(sfc + 8 * at, sdesc_sf(s.sf[slot][0] + 512 * at));
                        tc_cp_sf(sfc + 8 * at + 4, sdesc_sf(s.sf[slot][1] + 512 * at));
                        tc_cp_sf(sfc + 8 * kAt + 4 * at, sdesc_sf(s.sf[slot][2] + 512 * at));
                    }
                    const uint64_t dt = sdesc_sw128(s.b[slot]), dw = sdesc_sw128(s.a[slot][0]);  // a[slot][0..1]: 256 rows
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {  // 32 bytes of every row per MMA
                        const uint32_t acc = (kt | ks) != 0;
                        if (AF == 8) {  // K 32: one scale per row, byte ks of the stage's atom
                            const uint32_t id = idesc_sf_ids(idesc, ks, ks), sel = (uint32_t)ks << 30;
                            tc_mma_mx(tmem, dt + 2 * ks, dw + 2 * ks, id, (sfc + 8) | sel, sfc | sel, acc);
                        } else {        // K 64: scales 2 (ks % 2), + 1 of atom ks / 2
                            const uint32_t b0 = 2 * (ks & 1), at = ks >> 1;
                            const uint32_t id = idesc_sf_ids(idesc, b0, b0), sel = b0 << 30;
                            tc_mma_mxf4(tmem, dt + 2 * ks, dw + 2 * ks, id, (sfc + 8 * kAt + 4 * at) | sel,
                                        (sfc + 8 * at) | sel, acc);
                        }
                    }
                    tc_commit(&s.empty[slot]);  // frees the stage once these MMAs finish
                }
                if (!ok) { tc_fail(a, s); break; }
                tc_commit(&s.acc_full);
            }
            tc_commit(&s.mma_done);
            mbar_wait(&s.mma_done, 0);
        }
    } else {
        // ------------------------------ epilogue ------------------------------
        // TMEM lane = token of the tile (this warp: tokens 32 q .. 32 q + 31),
        // column = weight row: gate/up g at 0..127 and u at 128..255, down the
        // tile's 256 output features. Warp half h takes F rows 64 h .. +63
        // (gate/up) or features 128 h .. +127 (down).
        const int q = warp & 3;              // TMEM lane quarter this warp may access
        const int half = (warp - 2) >> 2;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        const int t = 32 * q + lane;         // this thread's token in the tile
        int lw = 0;
        // control flow stays warp-uniform: tcgen05.ld is a warp-collective
        for (int w = blockIdx.x; w < n_work; w += gridDim.x, ++lw) {
            if (__shfl_sync(0xffffffffu, s.abort, 0)) break;
            const Work wk = work_of(w, ft, s.ustart, a.E, a.offsets);
            const bool ok = mbar_wait(&s.acc_full, lw & 1);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) tc_fail(a, s);
                break;
            }
            tc_fence_after();
            const bool busy = 32 * q < wk.nvalid;  // warp-uniform: any valid token in this quarter
            const bool valid = t < wk.nvalid;
            // Pull this warp's columns out of TMEM (four loads and one wait; gate/up:
            // its g and u columns), then hand the accumulator back before the slow
            // part, so the next tile's MMAs overlap the SwiGLU, the requantisation
            // and the stores.
            float v[GU ? 64 : 128];
            uint32_t g0[32], g1[32], u0[32], u1[32];  // gate/up: raw g, u, then h in g0, g1
            if (busy) {
                if (GU) {
                    tmem_ld32(lane_base + 32 * (2 * half), g0);
                    tmem_ld32(lane_base + 32 * (2 * half + 1), g1);
                    tmem_ld32(lane_base + 128 + 32 * (2 * half), u0);
                    tmem_ld32(lane_base + 128 + 32 * (2 * half + 1), u1);
                    tmem_wait_ld();
                } else {  // the tile's four 32-column chunks of this warp's 128 features
                    tmem_ld32(lane_base + 128 * half, g0);
                    tmem_ld32(lane_base + 128 * half + 32, g1);
                    tmem_ld32(lane_base + 128 * half + 64, u0);
                    tmem_ld32(lane_base + 128 * half + 96, u1);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        v[i] = __uint_as_float(g0[i]);
                        v[32 + i] = __uint_as_float(g1[i]);
                        v[64 + i] = __uint_as_float(u0[i]);
                        v[96 + i] = __uint_as_float(u1[i]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.acc_empty);
            if (!busy) continue;
            if (GU) {
                // h = silu(g) u, in place (fewer live registers than a separate array)
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float ga = __uint_as_float(g0[i]), gb = __uint_as_float(g1[i]);
                    g0[i] = __float_as_uint(__fdividef(ga, 1.0f + __expf(-ga)) * __uint_as_float(u0[i]));
                    g1[i] = __float_as_uint(__fdividef(gb, 1.0f + __expf(-gb)) * __uint_as_float(u1[i]));
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    v[i] = __uint_as_float(g0[i]);
                    v[32 + i] = __uint_as_float(g1[i]);
                }
                // MXFP8 (MXFP4) along F: each block of 32 is 32 of this thread's
                // values; scale 2^(floor(log2 amax) - 8 (2)), an all-zero block
                // gets scale byte 127 (and codes of +-0)
                const int64_t atom = (((int64_t)s.ustart[wk.e] + wk.j) * (a.Nw / kTile) + wk.f) * 512;
                uint8_t *hrow = a.h8 + (int64_t)(wk.row0 + t) * (a.Nw * AF / 8) + (wk.f * kTile + 64 * half) * AF / 8;
#pragma unroll
                for (int bb = 0; bb < 2; ++bb) {
                    uint32_t amax = 0;
#pragma unroll
                    for (int i = 0; i < 32; ++i) amax = max(amax, __float_as_uint(v[32 * bb + i]) & 0x7FFFFFFFu);
                    int se = 0;
                    float sc = 0.0f;
                    if (amax != 0u) {
                        const int ee = floor_log2_f32(__uint_as_float(amax)) - (AF == 8 ? 8 : 2);
                        se = ee < -127 ? -127 : (ee > 127 ? 127 : ee);
                        sc = pow2_neg(se);
                    }
                    if (AF == 8) {
                        uint32_t pk[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            pk[i] = f32x2_to_e4m3x2(v[32 * bb + 4 * i] * sc, v[32 * bb + 4 * i + 1] * sc) |
                                    f32x2_to_e4m3x2(v[32 * bb + 4 * i + 2] * sc, v[32 * bb + 4 * i + 3] * sc) << 16;
                        if (valid) {
                            uint4 *dst = reinterpret_cast<uint4 *>(hrow + 32 * bb);
                            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                        }
                    } else {
                        uint32_t pk[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            pk[i] = e2m1x8(&v[32 * bb + 8 * i], sc);
                        if (valid) *reinterpret_cast<uint4 *>(hrow + 16 * bb) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                    if (valid) a.hsf[atom + sf_atom_byte(t, 2 * half + bb)] = (uint8_t)(se + 127);
                }
            } else if (valid) {
                const int64_t o0 = (int64_t)(wk.row0 + t) * a.Nw + wk.f * 2 * kTile + 128 * half;
                if (a.out16) {
                    uint4 *dst = reinterpret_cast<uint4 *>(a.out16 + o0);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        dst[i] = make_uint4(bf16x2(v[8 * i], v[8 * i + 1]), bf16x2(v[8 * i + 2], v[8 * i + 3]),
                                            bf16x2(v[8 * i + 4], v[8 * i + 5]), bf16x2(v[8 * i + 6], v[8 * i + 7]));
                } else {
                    float4 *dst = reinterpret_cast<float4 *>(a.out + o0);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// CTA 0: token tiles per expert (ceil(count / 128)) and their exclusive
// prefix. The other CTAs invert perm over the rows that hold a slot
// (offsets[E] of them; fewer than S only when some slot had no valid expert):
// row_of[slot] = the row holding the slot (row_of enters filled with -1, so a
// slot no row names stays -1).
__global__ void __launch_bounds__(1024) tc_plan_kernel(const int32_t *__restrict__ offsets, int E,
                                                       int32_t *__restrict__ ustart,
                                                       const int32_t *__restrict__ perm, int S,
                                                       int32_t *__restrict__ row_of, int *err) {
    if (blockIdx.x > 0) {
        const int i = (blockIdx.x - 1) * blockDim.x + threadIdx.x;
        if (i < min(S, offsets[E])) {
            const int slot = perm[i];
            if ((unsigned)slot < (unsigned)S) row_of[slot] = i;
            else set_device_error(err, MOE_DEVERR_PERM);
        }
        return;
    }
    __shared__ int wsum[32];
    const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
    const int nt = e < E ? (offsets[e + 1] - offsets[e] + kTile - 1) / kTile : 0;
    int incl = nt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int v = wsum[lane], w = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += t;
        }
        wsum[lane] = w - v;  // exclusive warp prefix
    }
    __syncthreads();
    const int excl = wsum[warp] + incl - nt;
    if (e < E) ustart[e] = excl;
    if (e == E - 1) ustart[E] = excl + nt;
}

// One warp per token: its x row becomes MXFP8 (AF 8: E4M3 codes) or MXFP4
// (AF 4: E2M1 codes, two per byte) once, with E8M0 scales per 32 along d (the
// OCP rule: scale exponent floor(log2 amax) - 8 or - 2, RNE, saturating; an
// all-zero block gets scale 127 and zero codes), and the codes go to each of
// the token's k rows in expert order, the scales to those rows' token-tile
// atoms. x is read once per token instead of once per row.
template <int AF>
__global__ void __launch_bounds__(256) tc_gather_quant_kernel(const uint16_t *__restrict__ x,
                                                              const int32_t *__restrict__ offsets,
                                                              const int32_t *__restrict__ row_of,
                                                              const int32_t *__restrict__ ustart, int T, int E,
                                                              int k, int d, uint8_t *__restrict__ x8,
                                                              uint8_t *__restrict__ xsf, int *err) {
    __shared__ int s_row[8][32], s_rt[8][32];
    __shared__ int64_t s_atom[8][32];
    const int wl = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + wl;
    if (t >= T) return;
    const int S = T * k;
    if (lane < k) {  // slot (t, lane): its row, the row's token-tile atom base and place in the tile
        int row = row_of[(int64_t)t * k + lane];
        const int nrows = min(S, offsets[E]);
        // a slot without a row is an error only when every slot should have one
        // (fewer rows: slots of experts another rank or another cache wave runs)
        if (row >= nrows || (row < 0 && nrows == S)) set_device_error(err, MOE_DEVERR_PERM);
        if (row < 0 || row >= nrows) {
            row = -1;
        } else {
            const int e = expert_of_row(offsets, E, row), r = row - offsets[e];
            s_atom[wl][lane] = ((int64_t)ustart[e] + r / kTile) * (d / kTile);
            s_rt[wl][lane] = r % kTile;
        }
        s_row[wl][lane] = row;
    }
    __syncwarp();
    const uint16_t *xr = x + (int64_t)t * d;
    for (int c0 = 0; c0 < d; c0 += 4 * 256) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {  // four loads in flight
            const int i0 = c0 + 256 * u + 8 * lane;
            v[u] = i0 < d ? __ldg(reinterpret_cast<const uint4 *>(xr + i0)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i0 = c0 + 256 * u + 8 * lane;
            const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            float f[8], amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                f[2 * i] = __uint_as_float(w[i] << 16);
                f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
                amax = fmaxf(amax, fmaxf(fabsf(f[2 * i]), fabsf(f[2 * i + 1])));
            }
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            uint32_t lo = 0, hi = 0, sb = 127;
            if (amax > 0.0f) {
                int se = floor_log2_f32(amax) - (AF == 8 ? 8 : 2);
                se = se < -127 ? -127 : (se > 127 ? 127 : se);
                sb = (uint32_t)(se + 127);
                const float sc = pow2_neg(se);
                if (AF == 8) {
                    lo = f32x2_to_e4m3x2(f[0] * sc, f[1] * sc) | f32x2_to_e4m3x2(f[2] * sc, f[3] * sc) << 16;
                    hi = f32x2_to_e4m3x2(f[4] * sc, f[5] * sc) | f32x2_to_e4m3x2(f[6] * sc, f[7] * sc) << 16;
                } else {
                    lo = e2m1x8(f, sc);
                }
            }
            if (i0 >= d) continue;
            const int b = i0 / 32;
            for (int j = 0; j < k; ++j) {
                const int row = s_row[wl][j];
                if (row < 0) continue;
                if (AF == 8) *reinterpret_cast<uint2 *>(x8 + (int64_t)row * d + i0) = make_uint2(lo, hi);
                else *reinterpret_cast<uint32_t *>(x8 + (int64_t)row * (d / 2) + i0 / 2) = lo;
                if ((lane & 3) == 0) xsf[(s_atom[wl][j] + b / 4) * 512 + sf_atom_byte(s_rt[wl][j], b % 4)] = (uint8_t)sb;
            }
        }
    }
}

int tc_num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

cudaError_t tc_set_attrs() {
    static std::atomic<bool> done[64];  // per device; a repeated set-up from racing threads is harmless
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    cudaError_t e;
    void (*const kernels[4])(TcArgs) = {tc_ffn_kernel<kModeGU, 8>, tc_ffn_kernel<kModeDN, 8>,
                                        tc_ffn_kernel<kModeGU, 4>, tc_ffn_kernel<kModeDN, 4>};
    for (auto k : kernels)
        if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemBytes))) return e;
    done[dev].store(true, std::memory_order_release);
    return cudaSuccess;
}

}  // namespace

bool tc_path_applies(const moe_dims &d) {
    // K per stage: 128 (w4a8) or 256 (w4a4) for both GEMMs (K = d_model, d_ff)
    const int ks = d.act == MOE_A_MXFP4 ? 2 * kTile : kTile;
    return d.wfmt == MOE_W_MXFP4 && (d.act == MOE_A_MXFP8 || d.act == MOE_A_MXFP4) && d.d_model % (2 * kTile) == 0 &&
           d.d_model % ks == 0 && d.d_ff % ks == 0 && d.E <= kTcMaxE && d.T >= 1;
}

// Routed expert FFN (MXFP4 weights; w4a8 or w4a4) on the tensor cores: plan,
// gather + quantise, gate/up GEMM with SwiGLU and MXFP8 (MXFP4)
// requantisation, down GEMM.
cudaError_t launch_tc_ffn(const moe_dims &d, const moe_weights &w, const uint16_t *x, const int32_t *offsets,
                          const int32_t *perm, float *out_rows, uint8_t *ws, const WsLayout &L, cudaStream_t s,
                          bool rows_bf16) {
    const int S = d.T * d.k;
    if (S == 0) return cudaSuccess;
    cudaError_t e = tc_set_attrs();
    if (e != cudaSuccess) return e;
    const Mxfp4Layout L1 = mxfp4_layout(d, MOE_MAT_W1), L2 = mxfp4_layout(d, MOE_MAT_W2);
    const uint8_t *p1 = static_cast<const uint8_t *>(w.w1), *p3 = static_cast<const uint8_t *>(w.w3),
                  *p2 = static_cast<const uint8_t *>(w.w2);
    int32_t *ustart = reinterpret_cast<int32_t *>(ws + L.ustart);
    uint8_t *gx8 = ws + L.gx8, *gxsf = ws + L.gxsf, *h8 = ws + L.h8, *hsf = ws + L.ghsf;

    TcArgs g;
    memset(&g, 0, sizeof g);
    TcArgs dn;
    memset(&dn, 0, sizeof dn);
    const uint64_t r13 = (uint64_t)d.E * d.d_ff, r2 = (uint64_t)d.E * d.d_model;
    const bool a4 = d.act == MOE_A_MXFP4;
    bool ok;
    if (a4)  // packed E2M1 on both sides: byte boxes of 128 x 128
        ok = make_tile_map_u8(&g.wa, p1 + L1.codes, r13, d.d_model / 2, kTile) &&
             make_tile_map_u8(&g.wb, p3 + L1.codes, r13, d.d_model / 2, kTile) &&
             make_tile_map_u8(&g.act, gx8, S, d.d_model / 2, kTile) &&
             make_tile_map_u8(&dn.wa, p2 + L2.codes, r2, d.d_ff / 2, kTile) &&
             make_tile_map_u8(&dn.wb, p2 + L2.codes, r2, d.d_ff / 2, kTile) &&
             make_tile_map_u8(&dn.act, h8, S, d.d_ff / 2, kTile);
    else     // E2M1 weights expanded to a byte per element beside E4M3 tokens
        ok = make_tile_map_e2m1(&g.wa, p1 + L1.codes, r13, d.d_model, kTile) &&
             make_tile_map_e2m1(&g.wb, p3 + L1.codes, r13, d.d_model, kTile) &&
             make_tile_map_u8(&g.act, gx8, S, d.d_model, kTile) &&
             make_tile_map_e2m1(&dn.wa, p2 + L2.codes, r2, d.d_ff, kTile) &&
             make_tile_map_e2m1(&dn.wb, p2 + L2.codes, r2, d.d_ff, kTile) &&
             make_tile_map_u8(&dn.act, h8, S, d.d_ff, kTile);
    if (!ok) return cudaErrorInvalidValue;
    g.sfa = p1 + L1.stile; g.sfb = p3 + L1.stile; g.sfact = gxsf;
    g.offsets = offsets; g.ustart = ustart; g.E = d.E; g.Nw = d.d_ff; g.K = d.d_model;
    g.h8 = h8; g.hsf = hsf; g.err = device_error_word();
    dn.sfa = p2 + L2.stile; dn.sfb = p2 + L2.stile; dn.sfact = hsf;
    dn.offsets = offsets; dn.ustart = ustart; dn.E = d.E; dn.Nw = d.d_model; dn.K = d.d_ff;
    if (rows_bf16) dn.out16 = reinterpret_cast<uint16_t *>(out_rows);
    else dn.out = out_rows;
    dn.err = g.err;

    if ((e = launch_tc_gather(d, x, offsets, perm, ustart, reinterpret_cast<int32_t *>(ws + L.row_of), gx8, gxsf, s)))
        return e;
    const int grid = tc_num_sms();
    if (a4) {
        tc_ffn_kernel<kModeGU, 4><<<grid, kTcThreads, kTcSmemBytes, s>>>(g);
        tc_ffn_kernel<kModeDN, 4><<<grid, kTcThreads, kTcSmemBytes, s>>>(dn);
    } else {
        tc_ffn_kernel<kModeGU, 8><<<grid, kTcThreads, kTcSmemBytes, s>>>(g);
        tc_ffn_kernel<kModeDN, 8><<<grid, kTcThreads, kTcSmemBytes, s>>>(dn);
    }
    count_launches(2);
    return cudaGetLastError();
}

// The tensor-core path's activation staging: token-tile plan, slot -> row
// inverse of perm, and the MXFP8 (MXFP4) rows in expert order with their
// scale atoms (gx8 [S][d] ([S][d/2]), gxsf [tiles][d/128][512], ustart [E+1]).
cudaError_t launch_tc_plan(const moe_dims &d, const int32_t *offsets, const int32_t *perm, int32_t *ustart,
                           int32_t *row_of, cudaStream_t s) {
    const int S = d.T * d.k;
    if (S == 0) return cudaSuccess;
    cudaError_t e;
    if ((e = cudaMemsetAsync(row_of, 0xFF, (size_t)S * 4, s)) != cudaSuccess) return e;
    tc_plan_kernel<<<1 + (S + 1023) / 1024, 1024, 0, s>>>(offsets, d.E, ustart, perm, S, row_of, device_error_word());
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_tc_gather(const moe_dims &d, const uint16_t *x, const int32_t *offsets, const int32_t *perm,
                             int32_t *ustart, int32_t *row_of, uint8_t *gx8, uint8_t *gxsf, cudaStream_t s) {
    const int S = d.T * d.k;
    if (S == 0) return cudaSuccess;
    cudaError_t e;
    int *err = device_error_word();
    if ((e = launch_tc_plan(d, offsets, perm, ustart, row_of, s)) != cudaSuccess) return e;
    if (d.act == MOE_A_MXFP4)
        tc_gather_quant_kernel<4><<<(d.T + 7) / 8, 256, 0, s>>>(x, offsets, row_of, ustart, d.T, d.E, d.k, d.d_model,
                                                                gx8, gxsf, err);
    else
        tc_gather_quant_kernel<8><<<(d.T + 7) / 8, 256, 0, s>>>(x, offsets, row_of, ustart, d.T, d.E, d.k, d.d_model,
                                                                gx8, gxsf, err);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
