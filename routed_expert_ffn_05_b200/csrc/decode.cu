// Decode-sized expert FFN (T <= 8 tokens): one persistent weight-streaming
// kernel on tensor cores, HBM-bound.
//
// Each routed expert is a SwiGLU FFN over MXFP4 (or Q2_K) weights; the shared
// expert is bf16 ("DS4", dibi8.com, "Key architectural innovations" item 1;
// "DwarfStar", hysenlabs.com, "Model support and quantisation"). With at most
// 8 tokens per expert the layer is a stream over the touched experts'
// weights, so the kernel is built around keeping HBM busy:
//  - one CTA per SM with three roles: a producer thread moves weight tiles
//    HBM -> shared memory with TMA (16-32 KB boxes, 128-byte swizzled; the
//    E8M0 scale boxes 64-byte swizzled) through four mbarrier stages; sixteen
//    consumer warps split K and run mma.sync (16 weight rows x 8 tokens:
//    m16n8k16 f16 with fp32 accumulation for MXFP4, m16n8k32 integer for the
//    Q2_K main term); an epilogue warp sums the consumers' partial tiles
//    (double-buffered) and writes the outputs;
//  - the work is numbered in units (a unit: one or more stages the consumers
//    run back to back, then one hand-off to the epilogue): shared gate/up
//    (streamed while routing finishes), routed gate/up, then down units; a
//    down unit waits (bounded) on a per-expert count of finished gate/up
//    tiles. CTAs claim the work in chunks from one ticket counter, in unit
//    order: shared gate/up units one at a time, routed gate/up as one large
//    chunk per CTA's worth of three quarters of it and then pairs, down units
//    as contiguous cost-balanced ranges over seven eighths of them and then
//    pairs. Every unit a down unit waits for was
//    claimed earlier by a CTA that is running and finishes its earlier claims
//    first, so the kernel needs no co-residency of its CTAs (other work may
//    hold some SMs, or a second layer may run on another stream);
//  - the producer stores each stage's decoded unit next to its data, so the
//    consumers read one word instead of decoding unit numbers;
//  - MXFP4 codes become f16 with the hardware E2M1 conversion; the E8M0 block
//    scale is applied per 32-element block in fp32;
//  - gate/up uses all T tokens as the MMA's N dimension, so its activation
//    fragments are built once per CTA; the epilogue reduces only the columns
//    of the tokens routed to the expert;
//  - x enters f16 range through an exact per-token power of two; h, rounded to
//    bf16 as the layer specifies, gets the same treatment per row from its
//    maximum, recorded with an order-free atomic max;
//  - launches are chained with programmatic dependent launch;
//  - every wait is bounded (MOE_DEVERR_TIMEOUT instead of a hang).
// K is permuted inside each 32-block identically for weights and activations:
// lane q of a quad holds elements 8q..8q+7 of a block, which cover its MMA
// k-slots of both k16 steps.
#include <string.h>

#include <atomic>

#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "tma.h"

namespace moe {
namespace {

constexpr int kCW = 16;                   // consumer warps (each owns 1/16 of K)
constexpr int kProducer = kCW;            // warp index of the producer
constexpr int kEpilogue = kCW + 1;        // warp index of the epilogue warp
constexpr int kThreads = (kCW + 2) * 32;
constexpr int kStageW = 32768;            // weight tile bytes per stage
// Stages and per-stage scale / metadata bytes by weight format: MXFP4 needs
// 2 KB of E8M0 per stage, Q2_K 8 KB of sc|m bytes and 2 KB of (d, dmin).
template <int WF> struct Pipe {  // (five MXFP4 stages were measured: no gain over four)
    static constexpr int stages = 4;
    static constexpr int meta = WF == MOE_W_Q2K ? 10240 : 2048;
};
constexpr int kQDd = 8192;                // Q2_K: offset of the (d, dmin) pairs in a stage's metadata
constexpr int kMaxE = 1024;
constexpr int kMaxSeg = 256;              // active experts of a decode batch: min(E, T k) <= 8 x 32
// Partial tiles: element (matrix m, row r < 16, column c < 8) of a consumer
// warp's 16x8 tiles at m * 144 + r * 9 + c. One column over all 16 rows and
// both matrices then falls in 32 different banks (the epilogue reads by
// column); the consumers' fragment stores conflict at most 2-way.
constexpr int kRedM = 144, kRedR = 9;
constexpr int kD = 4096, kF = 2048;       // the dims this tiling is written for
// A routed gate/up unit: 32 rows of W1 and W3 over all K for MXFP4 (two
// 16-row halves of two stages each, one hand-off), 16 rows (one stage) for Q2_K.
template <int WF> constexpr int gu_rows() { return WF == MOE_W_Q2K ? 16 : 32; }
template <int WF> constexpr int gu_tiles() { return kF / gu_rows<WF>(); }  // units per routed expert
// A routed down unit: 64 W2 rows over all K (two stages of 32 rows) for
// MXFP4, 32 rows (one stage) for Q2_K; its partial tiles are 16 rows each.
// (A 64-row Q2_K unit in one stage, with three stages to make room for its
// partial tiles, measured 1% faster at T = 8 and 5% slower at T = 1.)
template <int WF> constexpr int dn_rows() { return WF == MOE_W_Q2K ? 32 : 64; }
template <int WF> constexpr int dn_parts() { return dn_rows<WF>() / 32; }
template <int WF> constexpr int dn_stages() { return dn_parts<WF>(); }
template <int WF> constexpr int dn_tiles() { return kD / dn_rows<WF>(); }
// A consumer warp's partial-tile buffer holds one unit's 16-row tiles: a
// routed gate/up unit's (two matrices per 16 rows) or a down unit's, whichever
// is more (the shared expert's units need two). Floats per warp.
template <int WF> constexpr int red_tiles() {
    return dn_rows<WF>() / 16 > 2 * gu_rows<WF>() / 16 ? dn_rows<WF>() / 16 : 2 * gu_rows<WF>() / 16;
}
template <int WF> constexpr int red_w() { return red_tiles<WF>() * kRedM; }
static_assert(red_tiles<MOE_W_MXFP4>() >= 2 && red_tiles<MOE_W_Q2K>() >= 2, "partial tiles");
constexpr int kDshTiles = kD / 16;        // shared-expert down tiles

// Work kinds: shared gate/up (bf16, 8 stages of K 512), routed gate/up (MXFP4,
// 2 stages of K 2048), shared down (bf16, 2 stages of K 1024), routed down
// (MXFP4: 64 rows over all K in two stages of 32; Q2_K: 32 rows, one stage).
enum { kGsh = 0, kGrt = 1, kDsh = 2, kDrt = 3 };

struct DecodeArgs {
    CUtensorMap m1c, m3c, m2c;  // routed MXFP4 codes or Q2_K quants, chunked + swizzled
    CUtensorMap m1s, m3s, m2s;  // routed MXFP4 row-major scales, or Q2_K sc|m bytes (chunked)
    CUtensorMap ms1, ms3, ms2;  // shared expert (bf16), chunked + swizzled
    CUtensorMap m1d, m3d, m2d;  // Q2_K (d, dmin) pairs, row-major
    int T, E, k, Fs;
    const int32_t *offsets, *perm;
    const uint16_t *x;       // [T][d] bf16
    const float2 *xscale;    // [T] (2^p_t, 2^-p_t): x * 2^-p_t fits f16
    uint16_t *h;             // routed hidden [S][F] bf16
    uint32_t *hmax;          // [S] bits of max |h|
    uint16_t *hs;            // shared hidden [T][Fs] bf16
    float *out_rows;         // [S][d]
    float *shared_out;       // [T][d]
    uint32_t *counters;      // [0] work ticket, [1] shared gate/up tiles done, [2+s] gate/up tiles done of active expert s
                             // (all zeroed by a memset before the first kernel of the layer)
    int *err;
};

template <int WF>
struct Smem {
    static constexpr int kStages = Pipe<WF>::stages;
    uint8_t w[kStages][kStageW];
    uint8_t s[kStages][Pipe<WF>::meta];
    float red[2][kCW][red_w<WF>()];  // partial 16x8 tiles per consumer warp (see put_partial)
    uint64_t full[kStages], empty[kStages], rfull[2], rempty[2];
    int meta_u[kStages], meta_k[kStages];  // unit of the stage, and the unit decoded (pack_unit)
    int rmeta[2];
    int seg_e[kMaxSeg];
    int n_seg;
    volatile int abort;
    // the epilogue warp's own tables: per active expert its first row, row
    // count and tokens; per token the x prescale
    int ep_rbase[kMaxSeg];
    uint8_t ep_cnt[kMaxSeg];
    uint8_t ep_tok[kMaxSeg][8];
    float ep_xs[8];
};
template <int WF> constexpr int smem_bytes() { return (int)sizeof(Smem<WF>) + 1024; }  // + alignment slack
static_assert(smem_bytes<MOE_W_MXFP4>() <= 227 * 1024 && smem_bytes<MOE_W_Q2K>() <= 227 * 1024,
              "decode kernel shared memory");

template <int WF>
__device__ __forceinline__ Smem<WF> &smem_ref(uint8_t *raw) {
    return *reinterpret_cast<Smem<WF> *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ uint4 ldg128(const void *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }

// bf16 rows are read by MMA row g from shared row sigma(g) (and sigma(g) + 8):
// with the 128-byte swizzle this keeps each quarter warp's 16-byte reads on
// distinct bank groups. The epilogue puts results back at row sigma(g).
__device__ __forceinline__ int sigma(int g) { return (g >> 1) | ((g & 1) << 2); }

struct Unit {
    int kind, seg, tile, nst;
};

// Warp-wide: the experts with rows (offsets[e + 1] > offsets[e]) in ascending
// order; f(segment, expert, first row, end row) runs on the lane that found
// each one. Loads 8 x 32 experts' offsets at a time. Returns the count.
template <typename F>
__device__ __forceinline__ int active_experts(const int32_t *offsets, int E, int lane, F f) {
    int n = 0;
    for (int b0 = 0; b0 < E; b0 += 256) {
        int lo[8], hi[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = b0 + 32 * j + lane;
            lo[j] = e < E ? __ldcg(&offsets[e]) : 0;
            hi[j] = e < E ? __ldcg(&offsets[e + 1]) : 0;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const bool act = hi[j] > lo[j];
            const unsigned m = __ballot_sync(0xffffffffu, act);
            if (act) f(n + __popc(m & ((1u << lane) - 1u)), b0 + 32 * j + lane, lo[j], hi[j]);
            n += __popc(m);
        }
    }
    return n;
}

// Unit numbering: [shared gate/up][routed gate/up][shared down][routed down].
// The shared gate/up units need no routing: they stream while the routing
// kernels run. The shared down units sit between the two routed phases, where
// they need no wait (every shared gate/up tile is long done) and cover the
// tail of the routed gate/up phase. A routed gate/up unit is 16 rows of W1 and
// W3 over all K: four stages of MXFP4 codes (two per 16 rows), or one stage
// of Q2_K quants (16 rows, half the bytes per row).
template <int WF> constexpr int gu_stages() { return WF == MOE_W_Q2K ? 1 : 4; }

template <int WF>
__device__ __forceinline__ Unit unit_of(int u, int usg, int n_seg, int usd) {
    if (u < usg) return Unit{kGsh, -1, u, 8};
    int r = u - usg;
    if (r < n_seg * gu_tiles<WF>()) return Unit{kGrt, r / gu_tiles<WF>(), r % gu_tiles<WF>(), gu_stages<WF>()};
    r -= n_seg * gu_tiles<WF>();
    if (r < usd) return Unit{kDsh, -1, r, 2};
    r -= usd;
    return Unit{kDrt, r / dn_tiles<WF>(), r % dn_tiles<WF>(), dn_stages<WF>()};
}

template <class S>
__device__ __forceinline__ void fail(const DecodeArgs &a, S &s) {
    set_device_error(a.err, MOE_DEVERR_TIMEOUT);
    s.abort = 1;
}

// Test hooks for the inter-CTA wait below (moe_debug_set_wait): a shorter
// limit, and extra tiles to wait for that no CTA ever publishes. Zero = off.
__device__ uint64_t g_dbg_wait_ns = 0;
__device__ uint32_t g_dbg_wait_extra = 0;

// Bounded wait until *p >= target (another CTA's release). Lane 0 polls with
// backoff; every lane then acquires for itself.
__device__ __forceinline__ bool wait_count(const uint32_t *p, uint32_t target, int lane, const volatile int *abort) {
    bool ok = true;
    if (lane == 0) {
        target += g_dbg_wait_extra;
        if (ld_acquire(p) < target) {
            const uint64_t lim = g_dbg_wait_ns ? g_dbg_wait_ns : kWaitLimitNs;
            const uint64_t t0 = globaltimer_ns();
            while (ld_acquire(p) < target) {
                if (*abort || globaltimer_ns() - t0 > lim) { ok = false; break; }
                __nanosleep(256);
            }
        }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) ld_acquire(p);
    return ok;
}

// A unit's fields in one word for the consumers: kind (2 bits), stages (4),
// tile (8), active-expert segment (11; 0 for the shared expert).
__device__ __forceinline__ int pack_unit(const Unit &un) {
    return un.kind | un.nst << 2 | un.tile << 6 | max(un.seg, 0) << 14;
}
__device__ __forceinline__ Unit unpack_unit(int p) { return Unit{p & 3, p >> 14, (p >> 6) & 255, (p >> 2) & 15}; }

template <class S>
__device__ __forceinline__ void arm(S &s, int slot, int u, const Unit &un, uint32_t tx) {
    s.meta_u[slot] = u;
    s.meta_k[slot] = pack_unit(un);
    mbar_arrive_expect_tx(&s.full[slot], tx);
}

// Shared-memory word loads at a 32-bit address plus a compile-time offset.
template <int OFF>
__device__ __forceinline__ uint32_t lds32_at(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1+%2];" : "=r"(v) : "r"(addr), "n"(OFF));
    return v;
}

// One 32-block of MXFP4 rows against B: `addr` is lane (g, q)'s code word of
// row g (16-byte unit of the block, swizzled, + 4 q); row g + 8 sits 1024
// bytes (8 rows of 128) further. sl / sh: the rows' E8M0 scale words, byte sj.
template <int OFF>
__device__ __forceinline__ void mxfp4_block(float acc[4], uint32_t addr, uint32_t sw_lo, uint32_t sw_hi, int sj,
                                            const uint32_t b[4]) {
    uint32_t al[4], ah[4];
    e2m1x8_to_f16x8(lds32_at<OFF>(addr), al);
    e2m1x8_to_f16x8(lds32_at<OFF + 1024>(addr), ah);
    float t[4];
    mma_f16_16816_z(t, al[0], ah[0], al[1], ah[1], b[0], b[1]);
    mma_f16_16816(t, al[2], ah[2], al[3], ah[3], b[2], b[3]);
    const float sl = e8m0_fast(sw_lo, sj), sh = e8m0_fast(sw_hi, sj);
    acc[0] = fmaf(sl, t[0], acc[0]);
    acc[1] = fmaf(sl, t[1], acc[1]);
    acc[2] = fmaf(sh, t[2], acc[2]);
    acc[3] = fmaf(sh, t[3], acc[3]);
}

// One 32-block (64 bytes: units 4*(kb%2)..+3 of chunk kb/2) of bf16 rows
// sigma(g), sigma(g) + 8 against B (bf16).
__device__ __forceinline__ void bf16_block(float acc[4], const uint8_t *box, int rows, int kb, int g, int q,
                                           const uint32_t b[4]) {
    const int r = sigma(g), c = kb >> 1, u = 4 * (kb & 1) + q;
    const uint4 r0 = lds128(box + swz_off(c, rows, r, u));
    const uint4 r1 = lds128(box + swz_off(c, rows, r + 8, u));
    mma_bf16_16816(acc, r0.x, r1.x, r0.y, r1.y, b[0], b[1]);
    mma_bf16_16816(acc, r0.z, r1.z, r0.w, r1.w, b[2], b[3]);
}

// C fragment -> partial tile (rows r, columns c at r * 9 + c); MMA rows g,
// g + 8 land at rows rg, rg + 8.
__device__ __forceinline__ void put_partial(float *r, int rg, int q, const float acc[4]) {
    r[rg * kRedR + 2 * q] = acc[0];
    r[rg * kRedR + 2 * q + 1] = acc[1];
    r[(rg + 8) * kRedR + 2 * q] = acc[2];
    r[(rg + 8) * kRedR + 2 * q + 1] = acc[3];
}

// Byte offset of scale word w (the E8M0 bytes of 32-blocks 4w .. 4w + 3) of
// row r in a 64-byte-swizzled scale box (rows of 64 bytes).
__device__ __forceinline__ int scale_off(int r, int w) { return r * 64 + ((((w >> 2) ^ (r >> 1)) & 3) << 4) + 4 * (w & 3); }

// bf16 pair -> f16 pair scaled by an exact power of two.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v, float sc) {
    return f32x2_to_f16x2(__uint_as_float(v << 16) * sc, __uint_as_float(v & 0xFFFF0000u) * sc);
}

__device__ __forceinline__ uint32_t warp_max_bits(uint32_t v) {
    uint32_t r;
    asm volatile("redux.sync.max.u32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(v));
    return r;
}

__device__ __forceinline__ float row_scale(uint32_t hm) {  // 2^p with max |h| * 2^-p in [2^14, 2^15)
    return ldexpf(1.0f, hm ? floor_log2_f32(__uint_as_float(hm)) - 14 : 0);
}

// ---- Q2_K ----
// The main term runs on integer MMAs (m16n8k32, u8 x s8 and u8 x u8 -> s32).
// A is sc q (<= 45) per byte: the lane's quant word (lane order, layout.h)
// shifted and masked to four bytes, times the sub-block scale sc in one 32-bit
// multiply (no carry crosses a byte). B is the activation as an integer
// X = round(x 2^-p), |X| < 2^15 (p puts the row's largest |x| in [2^14, 2^15),
// so every element within 2^7 of it is exact), split into a signed high byte
// and an unsigned low byte, X = 256 hi + lo. The super-block's sum_k sc q X is
// 256 c_hi + c_lo, exact in 32 bits (< 2^29); d scales it once in fp32.

// One super-block (16 sub-blocks of 16), or half of one (HALF 0: sub-blocks
// 0..7, HALF 1: 8..15; HALF -1: all), of 16 rows r0 + sigma(g), r0 + sigma(g)
// + 8 in each of two parts P[0], P[1] of Q2_K boxes (gate/up: the W1 and the W3
// box; down: two 16-row tiles of one box), in lockstep, so four MMA chains are
// in flight. A part's box: quants `rows` rows in 128-byte chunks; sc|m the same
// rows, chunked; dd `ddrow` bytes per row, 64-byte swizzled for a whole
// super-block (gate/up boxes), row-major for a half (down boxes). B holds the
// part's K steps of 32 (high bytes in B[i][0..1], low bytes in B[i][2..3]); bm
// the sub-block sums as f16 hi + lo parts (bm[0..1] hi, bm[2..3] lo). MMA row g
// reads shared row sigma(g), so a quarter warp's 16-byte quant loads fall on 8
// different bank groups; the partial tile puts it back at row sigma(g).
// acc[p] += d (sum_j sc_j q . X) - dmin (sum_j m_j Xsum_j) over the part.
struct Q2Part {
    const uint8_t *qs, *scm, *dd;
    int r0;
};
template <int HALF>
__device__ __forceinline__ void q2k_superblock2(float (*acc)[4], const Q2Part (&P)[2], int rows, int ddrow, int sb,
                                                int g, int q, const uint32_t (*B)[4], const uint32_t bm[4]) {
    constexpr int S0 = HALF == 1 ? 4 : 0, NS = HALF < 0 ? 8 : 4;
    int rg[2], rh[2];
    const uint8_t *qlp[2], *qhp[2], *slp[2], *shp[2];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        rg[p] = P[p].r0 + sigma(g);
        rh[p] = rg[p] + 8;
        qlp[p] = P[p].qs + swz_off((sb * 64) / 128, rows, rg[p], 4 * (sb & 1) + q);
        qhp[p] = P[p].qs + swz_off((sb * 64) / 128, rows, rh[p], 4 * (sb & 1) + q);
        slp[p] = P[p].scm + swz_off((sb * 16) / 128, rows, rg[p], sb % 8);
        shp[p] = P[p].scm + swz_off((sb * 16) / 128, rows, rh[p], sb % 8);
    }
    int chi[2][4], clo[2][4];
#pragma unroll
    for (int p = 0; p < 2; ++p)
#pragma unroll
        for (int i = 0; i < 4; ++i) chi[p][i] = clo[p][i] = 0;
#pragma unroll
    for (int w = S0 / 2; w < (S0 + NS) / 2; ++w) {  // quant word w of the lane and sc|m word w: K steps 2w, 2w + 1
        uint32_t ql[2], qh[2], sl[2], sh[2];
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            ql[p] = lds32(qlp[p] + 4 * w);
            qh[p] = lds32(qhp[p] + 4 * w);
            sl[p] = lds32(slp[p] + 4 * w);
            sh[p] = lds32(shp[p] + 4 * w);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int st = 2 * w + h, i = st - S0;   // K 32 st .. + 31: sub-blocks 2 st, 2 st + 1
            const int sft = 4 * h, sb8 = 16 * h;     // their quants: shifts 4h, 4h + 2; scales: bytes 2h, 2h + 1
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                const uint32_t a0 = ((ql[p] >> sft) & 0x03030303u) * ((sl[p] >> sb8) & 15u);
                const uint32_t a1 = ((qh[p] >> sft) & 0x03030303u) * ((sh[p] >> sb8) & 15u);
                const uint32_t a2 = ((ql[p] >> (sft + 2)) & 0x03030303u) * ((sl[p] >> (sb8 + 8)) & 15u);
                const uint32_t a3 = ((qh[p] >> (sft + 2)) & 0x03030303u) * ((sh[p] >> (sb8 + 8)) & 15u);
                mma_u8s8_16832(chi[p], a0, a1, a2, a3, B[i][0], B[i][1]);
                mma_u8u8_16832(clo[p], a0, a1, a2, a3, B[i][2], B[i][3]);
            }
        }
    }
    // minimum term: A = m of sub-blocks 2q, 2q+1 (k-slots 2q, 2q+1) and 2q+8, 2q+9
    // (bytes 2 (q % 2), + 1 of sc|m words q / 2 and 2 + q / 2); a half keeps only
    // its own sub-blocks
    auto mpair = [&](uint32_t w) {  // bytes 0, 1 of w -> their high nibbles as an f16 subnormal pair
        return ((w >> 4) & 0xFu) | ((w << 4) & 0xF0000u);
    };
    const int sh16 = 16 * (q & 1);
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        const uint32_t ma0 = HALF == 1 ? 0u : mpair(lds32(slp[p] + 4 * (q >> 1)) >> sh16);
        const uint32_t ma1 = HALF == 1 ? 0u : mpair(lds32(shp[p] + 4 * (q >> 1)) >> sh16);
        const uint32_t ma2 = HALF == 0 ? 0u : mpair(lds32(slp[p] + 8 + 4 * (q >> 1)) >> sh16);
        const uint32_t ma3 = HALF == 0 ? 0u : mpair(lds32(shp[p] + 8 + 4 * (q >> 1)) >> sh16);
        float tn[4];
        mma_f16_16816_z(tn, ma0, ma1, ma2, ma3, bm[0], bm[1]);
        mma_f16_16816(tn, ma0, ma1, ma2, ma3, bm[2], bm[3]);
        const uint8_t *dd = P[p].dd;
        const uint32_t dl = lds32(dd + (HALF < 0 ? scale_off(rg[p], sb) : rg[p] * ddrow + 4 * sb));
        const uint32_t dh = lds32(dd + (HALF < 0 ? scale_off(rh[p], sb) : rh[p] * ddrow + 4 * sb));
        // dmin: 2^24 undoes the subnormal encoding of m, 2^5 the sub-block-sum pre-scale
        const float d0 = __half2float(__ushort_as_half((uint16_t)(dl & 0xFFFF)));
        const float m0 = __half2float(__ushort_as_half((uint16_t)(dl >> 16))) * 536870912.0f;
        const float d1 = __half2float(__ushort_as_half((uint16_t)(dh & 0xFFFF)));
        const float m1 = __half2float(__ushort_as_half((uint16_t)(dh >> 16))) * 536870912.0f;
        acc[p][0] = fmaf(-m0, tn[0], fmaf(d0, __int2float_rn(256 * chi[p][0] + clo[p][0]), acc[p][0]));
        acc[p][1] = fmaf(-m0, tn[1], fmaf(d0, __int2float_rn(256 * chi[p][1] + clo[p][1]), acc[p][1]));
        acc[p][2] = fmaf(-m1, tn[2], fmaf(d1, __int2float_rn(256 * chi[p][2] + clo[p][2]), acc[p][2]));
        acc[p][3] = fmaf(-m1, tn[3], fmaf(d1, __int2float_rn(256 * chi[p][3] + clo[p][3]), acc[p][3]));
    }
}

// B fragments of one super-block, or half of one (HALF as above), of an
// activation row (bf16 at `row` = the super-block's first element, scaled by
// `inv` into integers X as described above): step i's k-slots 4q .. 4q + 3 of
// sub-blocks 2 (S0 + i) and 2 (S0 + i) + 1, high bytes in B[i][0..1], low bytes
// in B[i][2..3]; bm gets the sums (scaled by 2^-5) of X over sub-blocks 2q,
// 2q+1, 2q+8, 2q+9 that lie in the part (zero otherwise), each split into an
// f16 part and the f16 of its remainder (exact: the sums are integers below
// 2^19, and the minimum term nearly cancels the main term, so it needs them
// whole).
template <int HALF, bool CG>
__device__ __forceinline__ void q2k_load_b(const uint16_t *row, float inv, int q, uint32_t (*B)[4], uint32_t bm[4]) {
    constexpr int S0 = HALF == 1 ? 4 : 0, NS = HALF < 0 ? 8 : 4;
    int keep[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < NS; ++i) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int j = 2 * (S0 + i) + h;  // sub-block
            const uint16_t *src = row + 16 * j + 4 * q;
            const uint2 v = CG ? __ldcg(reinterpret_cast<const uint2 *>(src)) : __ldg(reinterpret_cast<const uint2 *>(src));
            const int X0 = __float2int_rn(__uint_as_float(v.x << 16) * inv);
            const int X1 = __float2int_rn(__uint_as_float(v.x & 0xFFFF0000u) * inv);
            const int X2 = __float2int_rn(__uint_as_float(v.y << 16) * inv);
            const int X3 = __float2int_rn(__uint_as_float(v.y & 0xFFFF0000u) * inv);
            // byte 1 (high) and byte 0 (low) of each 16-bit two's-complement X
            B[i][h] = __byte_perm(__byte_perm(X0, X1, 0x0051), __byte_perm(X2, X3, 0x0051), 0x5410);
            B[i][2 + h] = __byte_perm(__byte_perm(X0, X1, 0x0040), __byte_perm(X2, X3, 0x0040), 0x5410);
            int ps = (X0 + X1) + (X2 + X3);
            ps += __shfl_xor_sync(0xffffffffu, ps, 1);
            ps += __shfl_xor_sync(0xffffffffu, ps, 2);
            if (j < 8 && (j >> 1) == q) keep[j & 1] = ps;
            if (j >= 8 && ((j - 8) >> 1) == q) keep[2 + (j & 1)] = ps;
        }
    }
    float hi[4], lo[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float v = (float)keep[i] * 0.03125f;  // exact: |keep| < 2^19
        hi[i] = __half2float(__float2half_rn(v));
        lo[i] = v - hi[i];
    }
    bm[0] = f32x2_to_f16x2(hi[0], hi[1]);
    bm[1] = f32x2_to_f16x2(hi[2], hi[3]);
    bm[2] = f32x2_to_f16x2(lo[0], lo[1]);
    bm[3] = f32x2_to_f16x2(lo[2], lo[3]);
}

template <int WF>
__global__ void __launch_bounds__(kThreads, 1) decode_ffn_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr bool Q2 = WF == MOE_W_Q2K;
    constexpr int kStages = Pipe<WF>::stages, kStageS = Pipe<WF>::meta;
    extern __shared__ uint8_t smem_raw[];
    Smem<WF> &s = smem_ref<WF>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == kProducer * 32) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], kCW);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.rfull[i], kCW);  // one arrival per consumer warp
            mbar_init(&s.rempty[i], 1);
        }
        s.abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    grid_dep_launch();
    const int usg = a.Fs > 0 ? a.Fs / 16 : 0;  // shared gate/up units (no routing needed)
    const int usd = a.Fs > 0 ? kDshTiles : 0;
    // finished gate/up tiles, published per expert (and for the shared expert)
    // by the epilogue; a down unit waits only for its own expert's tiles
    uint32_t *sh_done = a.counters + 1, *seg_done = a.counters + 2;

    // ------------------------------ producer ------------------------------
    if (warp == kProducer) {
        int gi = 0;
        auto issue = [&](int u, const Unit &un) {
            int row0 = 0;
            if (un.kind == kGrt) row0 = s.seg_e[un.seg] * kF + gu_rows<WF>() * un.tile;
            if (un.kind == kDrt) row0 = s.seg_e[un.seg] * kD + dn_rows<WF>() * un.tile;
            for (int c = 0; c < un.nst && !s.abort; ++c, ++gi) {
                const int slot = gi % kStages;
                if (!mbar_wait(&s.empty[slot], ((gi / kStages) & 1) ^ 1, &s.abort)) { fail(a, s); return; }
                uint8_t *w = s.w[slot];
                uint8_t *sm = &s.s[0][0] + (size_t)slot * kStageS;  // the stage's scale / metadata bytes
                uint64_t *bar = &s.full[slot];
                switch (un.kind) {
                    case kGsh:
                        arm(s, slot, u, un, 2 * 16384);
                        tma_load_3d(w, &a.ms1, 0, 16 * un.tile, 8 * c, bar);
                        tma_load_3d(w + 16384, &a.ms3, 0, 16 * un.tile, 8 * c, bar);
                        break;
                    case kGrt:
                        if (Q2) {  // quants, sc|m bytes and (d, dmin) of 16 rows over all K
                            arm(s, slot, u, un, 2 * 16384 + 2 * 4096 + 2 * 1024);
                            tma_load_3d(w, &a.m1c, 0, row0, 0, bar);
                            tma_load_3d(w + 16384, &a.m3c, 0, row0, 0, bar);
                            tma_load_3d(sm, &a.m1s, 0, row0, 0, bar);
                            tma_load_3d(sm + 4096, &a.m3s, 0, row0, 0, bar);
                            tma_load_2d(sm + kQDd, &a.m1d, 0, row0, bar);
                            tma_load_2d(sm + kQDd + 1024, &a.m3d, 0, row0, bar);
                        } else {  // stage c: rows row0 + 16 (c / 2) .. + 15, K half c % 2
                            const int rr = row0 + 16 * (c >> 1), kh = c & 1;
                            arm(s, slot, u, un, 2 * 16384 + 2 * 1024);
                            tma_load_3d(w, &a.m1c, 0, rr, 8 * kh, bar);
                            tma_load_3d(w + 16384, &a.m3c, 0, rr, 8 * kh, bar);
                            tma_load_2d(sm, &a.m1s, 64 * kh, rr, bar);
                            tma_load_2d(sm + 1024, &a.m3s, 64 * kh, rr, bar);
                        }
                        break;
                    case kDsh:
                        arm(s, slot, u, un, 32768);
                        tma_load_3d(w, &a.ms2, 0, 16 * un.tile, 16 * c, bar);
                        break;
                    default:
                        if (Q2) {  // 32 rows of W2 over all K
                            arm(s, slot, u, un, 16384 + 4096 + 1024);
                            tma_load_3d(w, &a.m2c, 0, row0, 0, bar);
                            tma_load_3d(sm, &a.m2s, 0, row0, 0, bar);
                            tma_load_2d(sm + kQDd, &a.m2d, 0, row0, bar);
                        } else {  // rows row0 + 32 c .. + 31 of the unit
                            arm(s, slot, u, un, 32768 + 2048);
                            tma_load_3d(w, &a.m2c, 0, row0 + 32 * c, 0, bar);
                            tma_load_2d(sm, &a.m2s, 0, row0 + 32 * c, bar);
                        }
                }
            }
        };
        // Work tickets: [0, usg) are the shared gate/up units, one each; they
        // need no routing, so they are claimed before the grid dependency
        // resolves. The counter was zeroed before the routing kernels ran.
        uint32_t *ticket = a.counters;
        int t = 0;
        if (lane == 0) {
            prefetch_tensormap(&a.m1c);
            prefetch_tensormap(&a.m2c);
            t = (int)atomicAdd(ticket, 1u);
            while (t < usg && !s.abort) {
                const int nt = (int)atomicAdd(ticket, 1u);  // the next claim is fetched one unit ahead
                issue(t, unit_of<WF>(t, usg, 0, 0));
                t = nt;
            }
        }
        __syncwarp();
        grid_dep_wait();  // routing results and zeroed counters from here on
        const int n = active_experts(a.offsets, a.E, lane, [&](int sg, int e, int, int) {
            if (sg < kMaxSeg) s.seg_e[sg] = e;
        });
        if (n > kMaxSeg) {  // cannot happen for T <= 8, k <= 32; refuse rather than overrun
            if (lane == 0) fail(a, s);
            return;
        }
        if (lane != 0) return;
        s.n_seg = n;
        const int G = (int)gridDim.x;
        const int gu_end = usg + n * gu_tiles<WF>();
        // Routed gate/up tickets: G chunks of cb units that hold three quarters
        // of the work (one per CTA when all run at once), then chunks of kGrab
        // units, which even out CTAs that started late or ran slow.
        constexpr int kGrab = 2;
        const int R = n * gu_tiles<WF>();
        const int cb = (R - R / 4) / G;
        const int nb = cb >= kGrab ? G : 0;
        const int t_small = usg + nb, t_dn = t_small + (R - nb * cb + kGrab - 1) / kGrab;
        // Down tickets: G contiguous ranges of equal cost over the shared and
        // routed down units (shared tiles cost 2 stages, routed ones dn_stages)
        // that hold seven eighths of the work, so a CTA changes expert, and
        // reloads its h fragments, once or twice; then chunks of kGrabD units,
        // which even out CTAs that reached the down phase late.
        constexpr int kDst = dn_stages<WF>(), kGrabD = 2;
        const long long cost = 2ll * usd + (long long)n * dn_tiles<WF>() * kDst;
        const long long cost_big = cost - cost / 8;
        auto first = [&](long long cst) {
            return gu_end + (cst <= 2ll * usd ? (int)((cst + 1) / 2)
                                              : usd + (int)((cst - 2ll * usd + kDst - 1) / kDst));
        };
        const int dn_end = gu_end + usd + n * dn_tiles<WF>();
        const int u_small = first(cost_big);
        const int t_dsmall = t_dn + G;
        const int t_end = t_dsmall + (dn_end - u_small + kGrabD - 1) / kGrabD;
        while (t < t_end && !s.abort) {
            int u0, u1;
            if (t < usg) {
                u0 = t;
                u1 = t + 1;
            } else if (t < t_small) {
                u0 = usg + (t - usg) * cb;
                u1 = u0 + cb;
            } else if (t < t_dn) {
                u0 = usg + nb * cb + (t - t_small) * kGrab;
                u1 = min(u0 + kGrab, gu_end);
            } else if (t < t_dsmall) {
                u0 = first(cost_big * (t - t_dn) / G);
                u1 = first(cost_big * (t - t_dn + 1) / G);
            } else {
                u0 = u_small + (t - t_dsmall) * kGrabD;
                u1 = min(u0 + kGrabD, dn_end);
            }
            // The next chunk is claimed while this chunk's last unit is issued
            // (the ring keeps the consumers a few stages behind), not earlier:
            // a CTA must not sit on a second large chunk while others idle.
            int nt = -1;
            for (int u = u0; u < u1 && !s.abort; ++u) {
                if (u == u1 - 1) nt = (int)atomicAdd(ticket, 1u);
                issue(u, unit_of<WF>(u, usg, n, usd));
            }
            t = nt >= 0 ? nt : (int)atomicAdd(ticket, 1u);
        }
        if (!s.abort) {
            const int slot = gi % kStages;
            if (mbar_wait(&s.empty[slot], ((gi / kStages) & 1) ^ 1, &s.abort)) {
                s.meta_u[slot] = -1;
                mbar_arrive(&s.full[slot]);
                ++gi;
            } else {
                fail(a, s);
            }
        }
        for (int g = gi - kStages; g < gi; ++g)  // copies in flight finish before exit
            if (g >= 0) mbar_wait(&s.full[g % kStages], (g / kStages) & 1);
        return;
    }

    // ------------------------------ epilogue ------------------------------
    if (warp == kEpilogue) {
        // The shared gate/up units come first and need no routing; the
        // per-expert tables (same ascending order as the producer's list) are
        // built when the first other unit arrives.
        int n = -1;
        auto tables = [&]() {
            grid_dep_wait();
            n = active_experts(a.offsets, a.E, lane, [&](int sg, int, int r0, int r1) {
                if (sg < kMaxSeg) {
                    s.ep_rbase[sg] = r0;
                    s.ep_cnt[sg] = (uint8_t)(r1 - r0);
                }
            });
            if (n > kMaxSeg) return false;
            __syncwarp();
            for (int sg = lane; sg < n; sg += 32) {
                const int rb = s.ep_rbase[sg], cnt = s.ep_cnt[sg];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (i < cnt) s.ep_tok[sg][i] = (uint8_t)(__ldcg(&a.perm[rb + i]) / a.k);
            }
            if (lane < a.T) s.ep_xs[lane] = a.xscale[lane].x;
            __syncwarp();
            return true;
        };
        // gate/up tiles finished here and not yet published: shared, and routed of segment pseg
        uint32_t sh_fin = 0, r_fin = 0;
        int pseg = -1;
        auto publish = [&]() {  // this warp's h / hs writes, then the counts
            if (!sh_fin && !r_fin) return;
            __threadfence();
            __syncwarp();
            if (lane == 0) {
                if (sh_fin) atomicAdd(sh_done, sh_fin);
                if (r_fin) atomicAdd(seg_done + pseg, r_fin);
            }
            sh_fin = r_fin = 0;
        };
        int dseg = -1;
        float dsc = 1.f;        // lane i < 8: output scale of row i of segment dseg
        for (int ru = 0;; ++ru) {
            const int rb = ru & 1;
            if (!mbar_wait(&s.rfull[rb], (ru >> 1) & 1, &s.abort)) { fail(a, s); return; }
            const int m = s.rmeta[rb];
            if (m == -1) return;
            if (m == -2) {  // before this CTA's first down unit (or its end): publish everything
                publish();
                if (lane == 0) mbar_arrive(&s.rempty[rb]);
                continue;
            }
            if ((m >> 3) >= usg && n < 0 && !tables()) {
                if (lane == 0) fail(a, s);
                return;
            }
            const Unit un = unit_of<WF>(m >> 3, usg, n, usd);
            // Sum over the consumer warps of one column: lane l takes matrix
            // (or down row half) l / 16, row l % 16 (four chains for latency).
            constexpr int kRedW = red_w<WF>();
            const float *red = &s.red[rb][0][0] + (lane >> 4) * kRedM + (lane & 15) * kRedR;
            auto colsum = [&](int c, int tile_pair = 0) {  // tile pair p: 16-row tiles 2p, 2p + 1
                const float *rp = red + 2 * kRedM * tile_pair;
                float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
#pragma unroll
                for (int w = 0; w < kCW; w += 4) {
                    v0 += rp[w * kRedW + c];
                    v1 += rp[(w + 1) * kRedW + c];
                    v2 += rp[(w + 2) * kRedW + c];
                    v3 += rp[(w + 3) * kRedW + c];
                }
                return (v0 + v1) + (v2 + v3);
            };
            const int row = lane & 15;
            if (un.kind == kGsh || un.kind == kGrt) {
                // lanes 0..15: gate of rows 0..15, lanes 16..31: up (a routed
                // unit: per 16-row half p, tiles 2p (gate) and 2p + 1 (up))
                const int col = 16 * un.tile + row;
                if (un.kind == kGsh) {
                    for (int c = 0; c < a.T; ++c) {
                        const float v = colsum(c);
                        const float up = __shfl_down_sync(0xffffffffu, v, 16);
                        if (lane < 16) a.hs[(int64_t)c * a.Fs + col] = f32_to_bf16_rne(silu_f32(v) * up);
                    }
                    ++sh_fin;
                    publish();  // at once (one atomic per shared tile): nothing later waits on it
                } else {
                    const int rbase = s.ep_rbase[un.seg], cnt = s.ep_cnt[un.seg];
                    for (int i = 0; i < cnt; ++i) {  // the expert's rows; column = the row's token
                        const int tok = s.ep_tok[un.seg][i];
                        const float xs = s.ep_xs[tok];
                        uint32_t hmx = 0;
#pragma unroll
                        for (int p = 0; p < gu_rows<WF>() / 16; ++p) {
                            const float v = colsum(tok, p);
                            const float up = __shfl_down_sync(0xffffffffu, v, 16);
                            if (lane < 16) {
                                const uint32_t hb = f32_to_bf16_rne(silu_f32(v * xs) * (up * xs));
                                a.h[(int64_t)(rbase + i) * kF + gu_rows<WF>() * un.tile + 16 * p + row] = (uint16_t)hb;
                                hmx = max(hmx, (hb & 0x7FFFu) << 16);
                            }
                        }
                        const uint32_t mx = warp_max_bits(hmx);
                        if (lane == 0) atomicMax(&a.hmax[rbase + i], mx);
                    }
                    if (un.seg != pseg) {  // a new expert: the previous one's count goes out
                        publish();
                        pseg = un.seg;
                    }
                    ++r_fin;
                }
            } else if (un.kind == kDsh) {
                // one matrix: lanes 0..15 and 16..31 take alternate columns
                for (int c = lane >> 4; c < a.T; c += 2) {
                    const float *r0 = &s.red[rb][0][0] + row * kRedR + c;
                    float v0 = 0.f, v1 = 0.f;
#pragma unroll
                    for (int w = 0; w < kCW; w += 2) {
                        v0 += r0[w * red_w<WF>()];
                        v1 += r0[(w + 1) * red_w<WF>()];
                    }
                    a.shared_out[(int64_t)c * kD + 16 * un.tile + row] = v0 + v1;
                }
            } else {
                // lane = row of each 32-row part of the unit; columns = the expert's rows
                const int rbase = s.ep_rbase[un.seg], cnt = s.ep_cnt[un.seg];
                if (un.seg != dseg) {
                    dseg = un.seg;
                    dsc = lane < cnt ? row_scale(__ldcg(&a.hmax[rbase + lane])) : 1.f;
                }
#pragma unroll
                for (int p = 0; p < dn_parts<WF>(); ++p)
                    for (int i = 0; i < cnt; ++i) {
                        const float sc = __shfl_sync(0xffffffffu, dsc, i);
                        a.out_rows[(int64_t)(rbase + i) * kD + dn_rows<WF>() * un.tile + 32 * p + lane] =
                            colsum(i, p) * sc;
                    }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.rempty[rb]);
        }
    }

    // ------------------------------ consumers ------------------------------
    // Warp w owns 1/16 of K in every unit: shared gate/up 1 block of 32 per
    // stage (8 stages of K 512), routed MXFP4 gate/up 4 blocks per stage (2 of
    // K 2048), shared down 2 blocks per stage (2 of K 1024), routed MXFP4
    // down 4 blocks of each 32-row stage (K 2048), Q2_K gate/up one
    // super-block, Q2_K down half of one. B holds this warp's activation
    // fragments for the unit's kind.
    const int g = lane >> 2, q = lane & 3;
    uint32_t B[8][4];
    uint32_t Bm[4];             // Q2_K: sub-block sums (hi, lo)
    int bkind = -1, bseg = -2;  // what B holds
    bool dep = false;           // grid dependency resolved for this thread
    bool flushed = false;       // gate/up counts of this CTA published
    float acc[2][4];
    int ru = 0;
    // Shared-memory addresses that stay fixed over stages. MXFP4 code words of
    // this lane: block jj of the warp's K slice is 16-byte unit 4 (w & 1) + jj
    // of chunk w / 2, rows g (+ 8 at +1024); a down box has 32 rows per chunk.
    // The unit index is xor-swizzled with g, so its bits 4..5 vary with jj
    // only through jj ^ (g & 3).
    // (A down box's chunks hold 32 rows: its code word sits 2048 (w / 2) bytes
    // further than a gate/up box's. Scale rows g + 8 sit 512 bytes after row g:
    // the swizzle term depends on (row / 2) % 4 only.)
    const uint32_t w_base = smem_u32(s.w[0]);
    constexpr uint32_t kScaleBase = (uint32_t)(kStages * kStageW);  // s.s[0] - s.w[0]
    const uint32_t code_gu = (uint32_t)swz_off(warp >> 1, 16, g, 4 * (warp & 1)) + 4 * q;
    const uint32_t sc_lo = (uint32_t)scale_off(g, warp);
    auto code_off = [&](uint32_t base, int jj) { return base ^ ((uint32_t)jj << 4); };
    auto marker = [&](int m) {  // a hand-off without a tile: -1 end, -2 publish
        const int rb = ru & 1;
        if (!mbar_wait(&s.rempty[rb], ((ru >> 1) & 1) ^ 1, &s.abort)) return false;
        if (threadIdx.x == 0) s.rmeta[rb] = m;
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.rfull[rb]);
        ++ru;
        return true;
    };
    auto release = [&](int slot) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.empty[slot]);
    };
    int slot = 0;      // ring slot of the current stage
    uint32_t ph = 0;   // its full-barrier parity
    auto advance = [&]() {
        if (++slot == kStages) {
            slot = 0;
            ph ^= 1u;
        }
    };
    auto next_stage = [&]() {  // the unit's next stage: wait until its data is in
        advance();
        return mbar_wait(&s.full[slot], ph, &s.abort);
    };
    for (;; advance()) {
        if (!mbar_wait(&s.full[slot], ph, &s.abort)) { fail(a, s); return; }
        const int u = s.meta_u[slot];
        if (u < 0) {  // end of work: publish (if still due) and tell the epilogue
            if ((!flushed && !marker(-2)) || !marker(-1)) fail(a, s);
            return;
        }
        const Unit un = unpack_unit(s.meta_k[slot]);
        if (un.kind != kGsh && !dep) {  // the shared gate/up units need no routing
            grid_dep_wait();
            dep = true;
        }
        // B depends on the kind, and for down units on the expert (its h rows)
        const int useg = (un.kind == kDrt) ? un.seg : -1;
        if (un.kind != bkind || useg != bseg) {
            bkind = un.kind;
            bseg = useg;
            if (un.kind == kDsh || un.kind == kDrt) {  // every gate/up unit must be complete
                // before the first down unit, this CTA's own gate/up counts go out
                // (they all precede it in claim order)
                if (!flushed) {
                    if (!marker(-2)) { fail(a, s); return; }
                    flushed = true;
                }
                const bool ok = un.kind == kDsh ? wait_count(sh_done, (uint32_t)usg, lane, &s.abort)
                                                : wait_count(seg_done + un.seg, (uint32_t)gu_tiles<WF>(), lane, &s.abort);
                if (!ok) { fail(a, s); return; }
            }
            if (Q2 && un.kind == kGrt) {  // x: super-block `warp` of K
                const int tok = min(g, a.T - 1);
                q2k_load_b<-1, false>(a.x + (int64_t)tok * kD + 256 * warp, a.xscale[tok].y, q, B, Bm);
            } else if (Q2 && un.kind == kDrt) {  // h: half (warp & 1) of super-block warp / 2
                const int e = s.seg_e[un.seg];
                const int rbase = a.offsets[e], cnt = a.offsets[e + 1] - rbase;
                const int row = rbase + min(g, cnt - 1);
                const float sc = 1.0f / row_scale(__ldcg(&a.hmax[row]));
                const uint16_t *hr = a.h + (int64_t)row * kF + 256 * (warp >> 1);
                if (warp & 1) q2k_load_b<1, true>(hr, sc, q, B, Bm);
                else q2k_load_b<0, true>(hr, sc, q, B, Bm);
            } else if (un.kind == kGsh || un.kind == kGrt) {
                const bool sh = un.kind == kGsh;
                const int tok = min(g, a.T - 1);
                const float inv = sh ? 1.f : a.xscale[tok].y;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    // shared: stage j holds blocks 16 j .. +15 of K; this warp takes 16 j + w
                    // routed: stage j/4 holds blocks 64 (j/4) .. +63; this warp takes 4w .. 4w+3
                    const int kb = sh ? 16 * j + warp : 64 * (j / 4) + 4 * warp + (j & 3);
                    const uint4 v = ldg128(a.x + (int64_t)tok * kD + 32 * kb + 8 * q);
                    const uint32_t raw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) B[j][i] = sh ? raw[i] : bf16x2_to_f16x2(raw[i], inv);
                }
            } else if (un.kind == kDsh) {
                const int tok = min(g, a.T - 1);
#pragma unroll
                for (int j = 0; j < 4; ++j) {  // stage j/2 holds blocks 32 (j/2) .. +31; this warp 2w, 2w+1
                    const uint4 v = ldcg128(a.hs + (int64_t)tok * a.Fs + 32 * (32 * (j / 2) + 2 * warp + (j & 1)) + 8 * q);
                    B[j][0] = v.x; B[j][1] = v.y; B[j][2] = v.z; B[j][3] = v.w;
                }
            } else {
                const int e = s.seg_e[un.seg];
                const int rbase = a.offsets[e], cnt = a.offsets[e + 1] - rbase;
                const int row = rbase + min(g, cnt - 1);
                const float sc = 1.0f / row_scale(__ldcg(&a.hmax[row]));
#pragma unroll
                for (int j = 0; j < 4; ++j) {  // blocks 4w .. 4w+3 of K
                    const uint4 v = ldcg128(a.h + (int64_t)row * kF + 32 * (4 * warp + j) + 8 * q);
                    B[j][0] = bf16x2_to_f16x2(v.x, sc);
                    B[j][1] = bf16x2_to_f16x2(v.y, sc);
                    B[j][2] = bf16x2_to_f16x2(v.z, sc);
                    B[j][3] = bf16x2_to_f16x2(v.w, sc);
                }
            }
        }
#pragma unroll
        for (int m = 0; m < 2; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;
        // The unit's stages, in order (the producer issues them back to back).
        if (un.kind == kGsh) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                if (c > 0 && !next_stage()) { fail(a, s); return; }
                const uint8_t *st = s.w[slot];
#pragma unroll
                for (int m = 0; m < 2; ++m) bf16_block(acc[m], st + 16384 * m, 16, warp, g, q, B[c]);
                release(slot);
            }
        } else if (Q2 && un.kind == kGrt) {
            const uint8_t *st = s.w[slot], *ss = s.s[slot];
            const Q2Part P[2] = {{st, ss, ss + kQDd, 0}, {st + 16384, ss + 4096, ss + kQDd + 1024, 0}};
            q2k_superblock2<-1>(acc, P, 16, 64, warp, g, q, B, Bm);
            release(slot);
        } else if (Q2 && un.kind == kDrt) {
            const uint8_t *st = s.w[slot], *ss = s.s[slot];
            const Q2Part P[2] = {{st, ss, ss + kQDd, 0}, {st, ss, ss + kQDd, 16}};
            if (warp & 1) q2k_superblock2<1>(acc, P, 32, 32, warp >> 1, g, q, B, Bm);
            else q2k_superblock2<0>(acc, P, 32, 32, warp >> 1, g, q, B, Bm);
            release(slot);
        } else if (un.kind == kGrt) {
            // two 16-row halves of two stages of K 2048 each: W1 rows at +0, W3
            // rows at +16384; E8M0 scale word w of rows g, g + 8 (W3's 1024
            // bytes further). The partial tiles go out per half (tiles 2h: gate,
            // 2h + 1: up), so the buffer is claimed first.
            if (!mbar_wait(&s.rempty[ru & 1], ((ru >> 1) & 1) ^ 1, &s.abort)) { fail(a, s); return; }
            float *red = s.red[ru & 1][warp];
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                if (h > 0) {
                    if (!next_stage()) { fail(a, s); return; }
#pragma unroll
                    for (int m = 0; m < 2; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;
                }
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    if (c > 0 && !next_stage()) { fail(a, s); return; }
                    const uint32_t cw = w_base + (uint32_t)slot * kStageW;
                    const uint32_t cs = w_base + kScaleBase + (uint32_t)slot * kStageS + sc_lo;
                    uint32_t sw[2][2];
                    sw[0][0] = lds32_at<0>(cs);
                    sw[0][1] = lds32_at<512>(cs);
                    sw[1][0] = lds32_at<1024>(cs);
                    sw[1][1] = lds32_at<1536>(cs);
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const uint32_t ad = cw + code_off(code_gu, jj);
                        mxfp4_block<0>(acc[0], ad, sw[0][0], sw[0][1], jj, B[4 * c + jj]);
                        mxfp4_block<16384>(acc[1], ad, sw[1][0], sw[1][1], jj, B[4 * c + jj]);
                    }
                    release(slot);
                }
                put_partial(red + 2 * kRedM * h, g, q, acc[0]);
                put_partial(red + (2 * h + 1) * kRedM, g, q, acc[1]);
            }
        } else if (un.kind == kDsh) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                if (c > 0 && !next_stage()) { fail(a, s); return; }
                const uint8_t *st = s.w[slot];
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) bf16_block(acc[0], st, 16, 2 * warp + jj, g, q, B[2 * c + jj]);
                release(slot);
            }
        } else {
            // dn_stages stages of 32 W2 rows over all K (rows 16 t + g (+ 8) of
            // each); B (the expert's h rows) is the same for all of them. The
            // partial tiles go out per stage, so the buffer is claimed first.
            if (!mbar_wait(&s.rempty[ru & 1], ((ru >> 1) & 1) ^ 1, &s.abort)) { fail(a, s); return; }
            float *red = s.red[ru & 1][warp];
#pragma unroll
            for (int c = 0; c < dn_stages<WF>(); ++c) {
                if (c > 0) {
                    if (!next_stage()) { fail(a, s); return; }
#pragma unroll
                    for (int m = 0; m < 2; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;
                }
                const uint32_t cw = w_base + (uint32_t)slot * kStageW + 2048u * (uint32_t)(warp >> 1);
                const uint32_t cs = w_base + kScaleBase + (uint32_t)slot * kStageS + sc_lo;
                uint32_t sw[2][2];
                sw[0][0] = lds32_at<0>(cs);
                sw[0][1] = lds32_at<512>(cs);
                sw[1][0] = lds32_at<1024>(cs);
                sw[1][1] = lds32_at<1536>(cs);
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const uint32_t ad = cw + code_off(code_gu, jj);
                    mxfp4_block<0>(acc[0], ad, sw[0][0], sw[0][1], jj, B[jj]);
                    mxfp4_block<2048>(acc[1], ad, sw[1][0], sw[1][1], jj, B[jj]);
                }
                release(slot);
                put_partial(red + 2 * kRedM * c, g, q, acc[0]);
                put_partial(red + (2 * c + 1) * kRedM, g, q, acc[1]);
            }
        }
        // hand the unit (or tile) to the epilogue warp (routed MXFP4 units and
        // Q2_K down units have put their tiles in place already)
        const int rb = ru & 1;
        if (un.kind == kGsh || un.kind == kDsh || (Q2 && un.kind == kGrt) || (Q2 && un.kind == kDrt)) {
            if (!mbar_wait(&s.rempty[rb], ((ru >> 1) & 1) ^ 1, &s.abort)) { fail(a, s); return; }
            // bf16 and Q2_K tiles read rows sigma(g)
            const int rg = (Q2 || un.kind == kGsh || un.kind == kDsh) ? sigma(g) : g;
            put_partial(s.red[rb][warp], rg, q, acc[0]);
            if (un.kind != kDsh) put_partial(s.red[rb][warp] + kRedM, rg, q, acc[1]);
        }
        if (threadIdx.x == 0) s.rmeta[rb] = u * 8 + (un.nst - 1);
        __syncwarp();  // the warp's tile stores, then one arrival (release) for the warp
        if (lane == 0) mbar_arrive(&s.rfull[rb]);
        ++ru;
    }
}

// ---------------------------------------------------------------------------
// Decode routing: fixed-order fp32 logits (one CTA per expert, one warp per
// token, lane = chunk; CTA 0 also computes the per-token f16 prescale), then
// one CTA does top-k, softmax gates, histogram / scan / permutation and
// resets the FFN kernel's per-row h maxima.
// ---------------------------------------------------------------------------
// One CTA per expert, one warp per token: lane c runs the fma chain over
// chunk c (elements 128 c .. 128 c + 127) in element order, then the fixed
// butterfly across the chunks. The expert's router row is staged once per CTA
// in shared memory as [16][32 lanes] uint4; the token's x chunk stays in
// registers. The warps of CTA 0 also write the per-token x prescale.
__global__ void __launch_bounds__(256) decode_logits_kernel(const uint16_t *__restrict__ x,
                                                            const uint16_t *__restrict__ wr,
                                                            const float *__restrict__ bias, int T, int E,
                                                            float *__restrict__ logits, float2 *__restrict__ xscale) {
    __shared__ uint4 ws4[16 * 32];
    // the finalize kernel (and through it the FFN kernel, whose shared-expert
    // tiles need no routing) may launch at once: they wait for this grid
    // before reading anything it writes
    grid_dep_launch();
    const int t = threadIdx.x >> 5, lane = threadIdx.x & 31, e = blockIdx.x;
    constexpr int chunk = kD / 32;  // 128 elements = 16 uint4 per lane
    for (int i = threadIdx.x; i < 16 * 32; i += blockDim.x)
        cp_async_16(&ws4[i], wr + (int64_t)e * kD + (i & 31) * chunk + 8 * (i >> 5));
    uint4 xv[16];
#pragma unroll
    for (int v = 0; v < 16; ++v) xv[v] = ldg128(x + (int64_t)t * kD + lane * chunk + 8 * v);
    cp_async_wait_all();
    __syncthreads();
    if (e == 0) {  // 2^p with max|x_t| 2^-p in [2^14, 2^15)
        float mx = 0.f;
#pragma unroll
        for (int v = 0; v < 16; ++v) {
            const uint32_t r[4] = {xv[v].x, xv[v].y, xv[v].z, xv[v].w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(r[j] << 16)), fabsf(__uint_as_float(r[j] & 0xFFFF0000u))));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) {
            const int p = mx > 0.f ? floor_log2_f32(mx) - 14 : 0;
            xscale[t] = make_float2(ldexpf(1.0f, p), ldexpf(1.0f, -p));
        }
    }
    float acc = 0.f;
#pragma unroll
    for (int v = 0; v < 16; ++v) {
        const uint4 wq = ws4[v * 32 + lane];
        const uint32_t wa[4] = {wq.x, wq.y, wq.z, wq.w};
        const uint32_t xa[4] = {xv[v].x, xv[v].y, xv[v].z, xv[v].w};
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            acc = __fmaf_rn(__uint_as_float(xa[qq] << 16), __uint_as_float(wa[qq] << 16), acc);
            acc = __fmaf_rn(__uint_as_float(xa[qq] & 0xFFFF0000u), __uint_as_float(wa[qq] & 0xFFFF0000u), acc);
        }
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
    if (lane == 0) logits[(int64_t)t * E + e] = bias ? __fadd_rn(acc, bias[e]) : acc;
}

struct FinalizeArgs {
    int T, E, k;
    int ebase, El;  // this call's experts: ids [ebase, ebase + El) (the whole layer: 0, E)
    const float *logits;
    int32_t *idx, *counts, *offsets, *perm, *inv_perm;
    float *gates;
    uint32_t *hmax;
};

__global__ void __launch_bounds__(256) decode_finalize_kernel(const FinalizeArgs a) {
    __shared__ float lg[8 * kMaxE];
    __shared__ int hist[kMaxE];
    __shared__ int sidx[256];
    __shared__ int run[kMaxE];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T, E = a.E, k = a.k;
    grid_dep_launch();
    for (int i = threadIdx.x; i < T * k; i += blockDim.x) a.hmax[i] = 0u;
    grid_dep_wait();
    for (int base = 0; base < T * E; base += 8 * 256) {  // 8 loads in flight per thread
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = base + 256 * j + threadIdx.x;
            v[j] = i < T * E ? __ldcg(a.logits + i) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = base + 256 * j + threadIdx.x;
            if (i < T * E) lg[i] = v[j];
        }
    }
    for (int e = threadIdx.x; e < a.El; e += blockDim.x) hist[e] = run[e] = 0;
    __syncthreads();
    if (warp < T) {  // top-k + gates of token `warp`: lane holds experts lane + 32 i
        const float *l = lg + warp * E;
        const int my_e = topk_row(l, E, k, lane);
        const float my_l = lane < k ? l[my_e] : 0.f;
        const float l0v = __shfl_sync(0xffffffffu, my_l, 0);
        const float ex = lane < k ? expf(my_l - l0v) : 0.f;
        const float den = warp_sum(ex);
        if (lane < k) {
            a.idx[warp * k + lane] = my_e;
            a.gates[warp * k + lane] = ex / den;
            sidx[warp * k + lane] = my_e;
        }
    }
    __syncthreads();
    const int S = T * k, El = a.El;
    if (threadIdx.x < S) {
        const int e = sidx[threadIdx.x] - a.ebase;
        if (e >= 0 && e < El) atomicAdd(&hist[e], 1);
    }
    __syncthreads();
    if (warp == 0) {  // exclusive scan over this call's experts; lane owns [lane * per, (lane + 1) * per)
        const int per = (El + 31) / 32, e0 = lane * per, e1 = min(El, e0 + per);
        int tot = 0;
        for (int e = e0; e < e1; ++e) tot += hist[e];
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int off = incl - tot;
        for (int e = e0; e < e1; ++e) {
            const int c = hist[e];
            a.counts[e] = c;
            a.offsets[e] = off;
            hist[e] = off;  // first row of expert e
            off += c;
        }
        if (lane == 31) a.offsets[El] = incl;
    }
    __syncthreads();
    // stable rank of each slot among the earlier slots of its expert: within a
    // warp by matching lanes, across warps through a running count per expert
    for (int w0 = 0; w0 * 32 < S; ++w0) {
        if (warp == w0) {
            const int s0 = threadIdx.x;
            const int el = s0 < S ? sidx[s0] - a.ebase : -1;
            const bool in = el >= 0 && el < El;  // a slot of another rank's expert gets no row
            const int e = in ? el : -1 - lane;
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            if (in) {
                const int row = hist[e] + run[e] + __popc(peers & ((1u << lane) - 1u));
                a.perm[row] = s0;
                a.inv_perm[s0] = row;
            } else if (s0 < S) {
                a.inv_perm[s0] = -1;
            }
            __syncwarp();
            if (in && lane == 31 - __clz(peers)) run[e] += __popc(peers);
        }
        __syncthreads();
    }
}

// Stage-API entry (no routing in this call): the x prescale and the h maxima reset.
__global__ void __launch_bounds__(256) decode_prep_kernel(const uint16_t *__restrict__ x, int T, int S,
                                                          float2 *xscale, uint32_t *hmax) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < T) {
        float mx = 0.f;
        for (int i = lane; i < kD / 8; i += 32) {
            const uint4 v = ldg128(x + (int64_t)warp * kD + 8 * i);
            const uint32_t r[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(r[j] << 16)), fabsf(__uint_as_float(r[j] & 0xFFFF0000u))));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) {
            const int p = mx > 0.f ? floor_log2_f32(mx) - 14 : 0;
            xscale[warp] = make_float2(ldexpf(1.0f, p), ldexpf(1.0f, -p));
        }
    }
    for (int i = threadIdx.x; i < S; i += blockDim.x) hmax[i] = 0u;
}

int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

cudaError_t set_smem_attrs() {
    static std::atomic<bool> done[64];  // per device; a repeated set-up from racing threads is harmless
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(decode_ffn_kernel<MOE_W_MXFP4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  smem_bytes<MOE_W_MXFP4>())))
        return e;
    if ((e = cudaFuncSetAttribute(decode_ffn_kernel<MOE_W_Q2K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  smem_bytes<MOE_W_Q2K>())))
        return e;
    done[dev].store(true, std::memory_order_release);
    return cudaSuccess;
}

// Launch with programmatic stream serialization: the kernel may start while
// its predecessor in the stream finishes; it calls griddepcontrol.wait before
// reading that predecessor's results.
template <typename... P, typename... A>
cudaError_t launch_pdl(void (*k)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, A... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, args...);
}

}  // namespace

cudaError_t set_debug_wait(uint64_t limit_ns, uint32_t extra) {
    cudaError_t e = cudaMemcpyToSymbol(g_dbg_wait_ns, &limit_ns, sizeof limit_ns);
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_dbg_wait_extra, &extra, sizeof extra);
    return e;
}

bool decode_path_applies(const moe_dims &d) {
    // the tiling is written for d_model 4096, d_ff 2048 (and a shared d_ff of 2048)
    return d.T >= 1 && d.T <= 8 && (d.wfmt == MOE_W_MXFP4 || d.wfmt == MOE_W_Q2K) && d.act == MOE_A_BF16 &&
           d.d_model == kD &&
           d.d_ff == kF && (d.d_ff_shared == 0 || d.d_ff_shared == 2048) && d.E <= kMaxE;
}

bool decode_route_applies(const moe_dims &d) {
    return decode_path_applies(d) && d.route == MOE_ROUTE_SOFTMAX_TOPK && d.T * d.k <= 256;
}

// Decode routing: logits kernel + finalize kernel (top-k, permute, scratch
// reset for the FFN kernel). The logits kernel also writes the x prescale.
cudaError_t launch_decode_route(const moe_dims &d, const uint16_t *x, const moe_weights &w, int32_t *idx,
                                float *gates, int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv_perm,
                                uint8_t *ws, const WsLayout &L, cudaStream_t s, int ebase, int El) {
    cudaError_t e = set_smem_attrs();
    if (e != cudaSuccess) return e;
    float *logits = reinterpret_cast<float *>(ws + L.logits);
    // the FFN kernel's work ticket and tile counts start at zero; the ticket is
    // taken before the FFN kernel waits for these routing kernels, so it is
    // reset here, ahead of them in stream order
    if ((e = cudaMemsetAsync(ws + L.counters, 0, (size_t)(d.E + 2) * 4, s)) != cudaSuccess) return e;  // E >= El
    decode_logits_kernel<<<d.E, 32 * d.T, 0, s>>>(x, w.w_router, w.router_bias, d.T, d.E, logits,
                                                  reinterpret_cast<float2 *>(ws + L.xscale));
    FinalizeArgs f;
    f.T = d.T; f.E = d.E; f.k = d.k; f.logits = logits;
    f.ebase = ebase;
    f.El = El < 0 ? d.E : El;
    f.idx = idx; f.counts = counts; f.offsets = offsets; f.perm = perm; f.inv_perm = inv_perm; f.gates = gates;
    f.hmax = reinterpret_cast<uint32_t *>(ws + L.hmax);
    if ((e = launch_pdl(decode_finalize_kernel, dim3(1), dim3(256), 0, s, f)) != cudaSuccess) return e;
    count_launches(2);
    return cudaGetLastError();
}

// Routed + shared expert FFN for decode batches in one launch. `shared_out`
// may be null. `prepared`: the decode routing already ran on this workspace
// (x prescale, counters and h maxima reset); otherwise a memset and a small
// kernel do that first.
cudaError_t launch_decode_ffn(const moe_dims &d, const moe_weights &w, const uint16_t *x, const int32_t *offsets,
                              const int32_t *perm, float *out_rows, float *shared_out, uint8_t *ws,
                              const WsLayout &L, cudaStream_t s, bool prepared) {
    cudaError_t e = set_smem_attrs();
    if (e != cudaSuccess) return e;
    DecodeArgs a;
    memset(&a, 0, sizeof a);
    const uint8_t *p1 = static_cast<const uint8_t *>(w.w1), *p3 = static_cast<const uint8_t *>(w.w3),
                  *p2 = static_cast<const uint8_t *>(w.w2);
    const uint64_t r13 = (uint64_t)d.E * kF, r2 = (uint64_t)d.E * kD;
    const bool q2 = d.wfmt == MOE_W_Q2K;
    bool ok;
    if (q2) {  // quants (64 B per 256 weights), sc|m bytes (16 B), (d, dmin) pairs (4 B)
        const Q2kLayout L1 = q2k_layout(d, MOE_MAT_W1), L2 = q2k_layout(d, MOE_MAT_W2);
        ok = make_chunked_map(&a.m1c, p1 + L1.qs, r13, kD / 4, 16, 8) &&
             make_chunked_map(&a.m3c, p3 + L1.qs, r13, kD / 4, 16, 8) &&
             make_chunked_map(&a.m2c, p2 + L2.qs, r2, kF / 4, 32, 4) &&
             make_chunked_map(&a.m1s, p1 + L1.scm, r13, kD / 16, 16, 2) &&
             make_chunked_map(&a.m3s, p3 + L1.scm, r13, kD / 16, 16, 2) &&
             make_chunked_map(&a.m2s, p2 + L2.scm, r2, kF / 16, 32, 1) &&
             make_plain_map(&a.m1d, p1 + L1.dd, r13, kD / 64, kD / 64, 16, true) &&
             make_plain_map(&a.m3d, p3 + L1.dd, r13, kD / 64, kD / 64, 16, true) &&
             make_plain_map(&a.m2d, p2 + L2.dd, r2, kF / 64, kF / 64, 32);
    } else {
        const Mxfp4Layout L1 = mxfp4_layout(d, MOE_MAT_W1), L2 = mxfp4_layout(d, MOE_MAT_W2);
        ok = make_chunked_map(&a.m1c, p1 + L1.codes, r13, kD / 2, 16, 8) &&
             make_chunked_map(&a.m3c, p3 + L1.codes, r13, kD / 2, 16, 8) &&
             make_chunked_map(&a.m2c, p2 + L2.codes, r2, kF / 2, 32, 8) &&
             make_plain_map(&a.m1s, p1 + L1.srow, r13, kD / 32, 64, 16, true) &&
             make_plain_map(&a.m3s, p3 + L1.srow, r13, kD / 32, 64, 16, true) &&
             make_plain_map(&a.m2s, p2 + L2.srow, r2, kF / 32, 64, 32, true);
    }
    if (ok && shared_out)
        ok = make_chunked_map(&a.ms1, w.sw1, d.d_ff_shared, kD * 2, 16, 8) &&
             make_chunked_map(&a.ms3, w.sw3, d.d_ff_shared, kD * 2, 16, 8) &&
             make_chunked_map(&a.ms2, w.sw2, kD, d.d_ff_shared * 2, 16, 16);
    if (!ok) return cudaErrorInvalidValue;
    a.T = d.T; a.E = d.E; a.k = d.k;
    a.Fs = shared_out ? d.d_ff_shared : 0;
    a.offsets = offsets; a.perm = perm; a.x = x;
    a.xscale = reinterpret_cast<const float2 *>(ws + L.xscale);
    a.h = reinterpret_cast<uint16_t *>(ws + L.h);
    a.hmax = reinterpret_cast<uint32_t *>(ws + L.hmax);
    a.hs = reinterpret_cast<uint16_t *>(ws + L.sh_h);
    a.out_rows = out_rows;
    a.shared_out = shared_out;
    a.counters = reinterpret_cast<uint32_t *>(ws + L.counters);
    a.err = device_error_word();
    if (!prepared) {
        if ((e = cudaMemsetAsync(a.counters, 0, (size_t)(d.E + 2) * 4, s)) != cudaSuccess) return e;
        decode_prep_kernel<<<1, 256, 0, s>>>(x, d.T, d.T * d.k, reinterpret_cast<float2 *>(ws + L.xscale), a.hmax);
        count_launches(1);
    }
    e = q2 ? launch_pdl(decode_ffn_kernel<MOE_W_Q2K>, dim3(num_sms()), dim3(kThreads), smem_bytes<MOE_W_Q2K>(), s, a)
           : launch_pdl(decode_ffn_kernel<MOE_W_MXFP4>, dim3(num_sms()), dim3(kThreads), smem_bytes<MOE_W_MXFP4>(), s,
                        a);
    if (e != cudaSuccess) return e;
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
