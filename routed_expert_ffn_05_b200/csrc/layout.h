// Byte layouts of the packed weights and of the workspace (host + device).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "moe.h"

#ifdef __CUDACC__
#define MOE_HD __host__ __device__
#else
#define MOE_HD
#endif

namespace moe {

static inline int64_t al256(int64_t v) { return (v + 255) / 256 * 256; }

// Rows N and input dim K of one routed-expert matrix.
static inline void mat_shape(const moe_dims &d, int which, int64_t &N, int64_t &K) {
    if (which == MOE_MAT_W2) { N = d.d_model; K = d.d_ff; }
    else { N = d.d_ff; K = d.d_model; }
}

// Packed MXFP4 matrix: codes [E][N][K/2] (as canonical), scales row-major
// [E][N][K/32], and the same scales tiled for the tensor-core path:
// [E][N/128][K/128] atoms of 512 bytes, byte (n%32)*16 + ((n%128)/32)*4 + kb%4
// for row n and 32-block kb (the scale-factor order tcgen05.cp 32x128b.warpx4
// spreads over TMEM lanes).
struct Mxfp4Layout {
    int64_t N, K, E, codes, srow, stile, total;
};
static inline Mxfp4Layout mxfp4_layout(const moe_dims &d, int which) {
    Mxfp4Layout L;
    mat_shape(d, which, L.N, L.K);
    L.E = d.E;
    L.codes = 0;
    L.srow = al256(L.E * L.N * L.K / 2);
    L.stile = al256(L.srow + L.E * L.N * L.K / 32);
    L.total = al256(L.stile + L.E * L.N * L.K / 32);
    return L;
}
MOE_HD static inline int64_t mxfp4_tile_index(int64_t e, int64_t n, int64_t kb, int64_t N, int64_t K) {
    const int64_t atom = (e * (N / 128) + n / 128) * (K / 128) + kb / 4;
    return atom * 512 + (n % 32) * 16 + ((n % 128) / 32) * 4 + (kb % 4);
}

// Packed Q2_K matrix: quants [E][N][K/256][64], sc|m<<4 bytes [E][N][K/256][16],
// (d, dmin) fp16 pairs [E][N][K/256].
//
// The 64 quant bytes of a super-block are 16 32-bit words in "lane order" for
// the integer MMA m16n8k32 (K 32 = two sub-blocks per MMA): quant e (0..255;
// sub-block c = e / 16) sits in word 4 ((e % 16) / 4) + c / 4 at bit
// 8 (e % 4) + 2 (c % 4). Lane q of an MMA quad reads words 4q .. 4q + 3 (16
// bytes), which hold elements 4q .. 4q + 3 of every sub-block; word 4q + c / 4
// shifted right by 2 (c % 4) and masked with 0x03030303 gives those four
// quants of sub-block c as four bytes, the A-fragment order of the MMA.
struct Q2kLayout {
    int64_t N, K, E, qs, scm, dd, total;
};
MOE_HD static inline int q2k_word(int e) { return 4 * ((e % 16) / 4) + (e / 16) / 4; }
MOE_HD static inline int q2k_bit(int e) { return 8 * (e % 4) + 2 * ((e / 16) % 4); }

static inline Q2kLayout q2k_layout(const moe_dims &d, int which) {
    Q2kLayout L;
    mat_shape(d, which, L.N, L.K);
    L.E = d.E;
    const int64_t nsb = L.E * L.N * (L.K / 256);
    L.qs = 0;
    L.scm = al256(nsb * 64);
    L.dd = al256(L.scm + nsb * 16);
    L.total = al256(L.dd + nsb * 4);
    return L;
}

// Workspace regions (byte offsets), one layout for every entry point.
struct WsLayout {
    int64_t logits, rnorm, topk_idx, topk_w, counts, offsets, perm, inv_perm, blkcnt, blkbase;
    int64_t x8, xs, xscale, counters, h, hmax, h8, hs, out_rows, sh_h, sh_out;
    int64_t ustart, row_of, gx8, gxsf, ghsf, slot_of, idx_slot, total;
    int64_t nblk, max_tiles;
};
static const int kPermuteBlock = 256;  // slots per permute block

static inline WsLayout ws_layout(const moe_dims &d) {
    WsLayout w;
    const int64_t T = d.T, S = (int64_t)d.T * d.k, E = d.E, dm = d.d_model, F = d.d_ff;
    w.nblk = (S + kPermuteBlock - 1) / kPermuteBlock;
    int64_t o = 0;
    auto take = [&](int64_t bytes) { const int64_t r = o; o = al256(o + bytes); return r; };
    w.logits = take(T * E * 4);  // router logits (the tensor-core router: its approximate logits)
    w.rnorm = take(E * 4);       // router rows' 2-norms (tensor-core router)
    w.topk_idx = take(S * 4);
    w.topk_w = take(S * 4);
    w.counts = take(E * 4);
    w.offsets = take((E + 1) * 4);
    w.perm = take(S * 4);
    w.inv_perm = take(S * 4);
    w.blkcnt = take(w.nblk * E * 4);
    w.blkbase = take(w.nblk * E * 4);
    w.x8 = take(T * dm);
    w.xs = take(T * dm / 32);
    w.xscale = take(T * 8);
    w.counters = take((E + 2) * 4);  // work queue, shared gate/up done, per-expert done
    w.h = take(S * F * 4);
    w.hmax = take(S * 4);
    w.h8 = take(S * F);
    w.hs = take(S * F / 32);
    w.out_rows = take(S * dm * 4);
    const int64_t Fs = d.d_ff_shared > 0 ? d.d_ff_shared : 0;
    w.sh_h = take(T * Fs * 4);
    w.sh_out = take(T * dm * 4);
    // tensor-core path: token tiles of 128 rows per expert (at most
    // ceil(S / 128) + E of them), the slot -> row inverse of perm, gathered
    // MXFP8 rows, and scale atoms of 512 bytes per (token tile, 128-wide K block)
    w.max_tiles = (S + 127) / 128 + E;
    w.ustart = take((E + 1) * 4);
    w.row_of = take(S * 4);  // slot -> permuted row
    w.gx8 = take(S * dm);
    w.gxsf = take(w.max_tiles * (dm / 128) * 512);
    w.ghsf = take(w.max_tiles * (F / 128) * 512);
    // expert cache: expert -> slot map of the current wave, slot of every top-k entry
    w.slot_of = take(E * 4);
    w.idx_slot = take(S * 4);
    w.total = o;
    return w;
}

}  // namespace moe
