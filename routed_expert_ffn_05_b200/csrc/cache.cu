// Routed experts served from host memory through a cache of expert slots in
// HBM (moe_cache_create, moe_layer_cached).
//
// The pages run models larger than memory by keeping the non-routed weights
// resident and the routed experts in a cache that is filled from storage on a
// miss ("DwarfStar", hysenlabs.com, "Running models larger than memory with
// SSD streaming"; baiwuji.top/articles/174, "Core features" item 2). Here the
// store is pinned host memory (all E experts, packed layout) and the cache is
// `slots` experts in HBM (packed layout of `slots` experts); router and shared
// expert stay resident. One call:
//  1. routes in full on the GPU, copies the top-k ids to the host and waits
//     (the only synchronisation: the host must know which experts to fetch);
//  2. groups the experts the batch touches into waves of at most `slots`
//     (cached ones first), and per wave picks a slot for each missing expert
//     (least recently used among the slots this wave does not need) and copies
//     its pieces host -> device, one cudaMemcpyAsync per contiguous piece;
//  3. per wave: maps expert ids to slots on the device (others -> -1), permutes
//     over the slots (slots of other waves take no row), runs the expert FFN on
//     the slot weights and combines into y (the first wave writes y with the
//     shared expert, later waves add to it).
// With one wave the output is bit for bit moe_layer's through the staged path.
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <vector>

#include "common.cuh"
#include "kernels.h"

struct moe_expert_cache {
    moe_dims dims;  // the layer (E = all experts); T is per call
    int slots;
    const uint8_t *host[3];  // W1, W3, W2: packed for E experts, pinned host memory
    uint8_t *dev[3];         //             packed for `slots` experts, device memory
    // per matrix: up to three contiguous per-expert pieces (offset of the piece
    // of expert 0 in a packed matrix of E experts / of `slots` experts, bytes per expert)
    int64_t host_off[3][3], dev_off[3][3], piece[3][3];
    std::vector<int> slot_expert, expert_slot;
    std::vector<uint64_t> last_use;
    uint64_t tick = 0;
    int32_t *h_idx = nullptr;  // pinned: the call's top-k ids
    int32_t *h_map = nullptr;  // pinned: [waves][E] slot maps
    int max_waves = 0, idx_cap = 0;
    moe_cache_stats stats;
};

namespace moe {
namespace {

__global__ void cache_remap_kernel(const int32_t *__restrict__ idx, int S, int E, const int32_t *__restrict__ slot_of,
                                   int32_t *__restrict__ out) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= S) return;
    const int e = idx[i];
    out[i] = (e >= 0 && e < E) ? slot_of[e] : -1;
}

// The per-expert contiguous pieces of one packed matrix (see layout.h).
void pieces(const moe_dims &d, int which, int E, int64_t off[3], int64_t per[3]) {
    int64_t N, K;
    mat_shape(d, which, N, K);
    moe_dims de = d;
    de.E = E;
    if (d.wfmt == MOE_W_Q2K) {
        const Q2kLayout L = q2k_layout(de, which);
        off[0] = L.qs; off[1] = L.scm; off[2] = L.dd;
        per[0] = N * (K / 256) * 64; per[1] = N * (K / 256) * 16; per[2] = N * (K / 256) * 4;
    } else {
        const Mxfp4Layout L = mxfp4_layout(de, which);
        off[0] = L.codes; off[1] = L.srow; off[2] = L.stile;
        per[0] = N * K / 2; per[1] = N * K / 32; per[2] = N * K / 32;
    }
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_cache_create(const moe_dims *dims, int32_t slots, const void *host_w1, const void *host_w3,
                            const void *host_w2, void *dev_w1, void *dev_w3, void *dev_w2, moe_expert_cache **out) {
    if (!out) return MOE_ERR_INVALID_ARG;
    *out = nullptr;
    size_t probe = 0;
    moe_status st = moe_workspace_size(dims, &probe);  // validates dims
    if (st != MOE_OK) return st;
    if (slots < 1 || slots > dims->E || !host_w1 || !host_w3 || !host_w2 || !dev_w1 || !dev_w3 || !dev_w2)
        return MOE_ERR_INVALID_ARG;
    for (const void *p : {(const void *)dev_w1, (const void *)dev_w3, (const void *)dev_w2})
        if (reinterpret_cast<uintptr_t>(p) % 256) return MOE_ERR_INVALID_ARG;
    moe_expert_cache *c = new (std::nothrow) moe_expert_cache();
    if (!c) return MOE_ERR_CUDA;
    c->dims = *dims;
    c->slots = slots;
    c->host[0] = static_cast<const uint8_t *>(host_w1);
    c->host[1] = static_cast<const uint8_t *>(host_w3);
    c->host[2] = static_cast<const uint8_t *>(host_w2);
    c->dev[0] = static_cast<uint8_t *>(dev_w1);
    c->dev[1] = static_cast<uint8_t *>(dev_w3);
    c->dev[2] = static_cast<uint8_t *>(dev_w2);
    const int which[3] = {MOE_MAT_W1, MOE_MAT_W3, MOE_MAT_W2};
    for (int m = 0; m < 3; ++m) {
        pieces(*dims, which[m], dims->E, c->host_off[m], c->piece[m]);
        int64_t per[3];
        pieces(*dims, which[m], slots, c->dev_off[m], per);
    }
    c->slot_expert.assign(slots, -1);
    c->expert_slot.assign(dims->E, -1);
    c->last_use.assign(slots, 0);
    c->max_waves = (dims->E + slots - 1) / slots;
    memset(&c->stats, 0, sizeof c->stats);
    if (cudaMallocHost(reinterpret_cast<void **>(&c->h_map), (size_t)c->max_waves * dims->E * 4) != cudaSuccess) {
        delete c;
        return MOE_ERR_CUDA;
    }
    *out = c;
    return MOE_OK;
}

moe_status moe_cache_destroy(moe_expert_cache *c) {
    if (!c) return MOE_OK;
    cudaFreeHost(c->h_idx);
    cudaFreeHost(c->h_map);
    delete c;
    return MOE_OK;
}

moe_status moe_cache_get_stats(const moe_expert_cache *c, moe_cache_stats *s) {
    if (!c || !s) return MOE_ERR_INVALID_ARG;
    *s = c->stats;
    return MOE_OK;
}

moe_status moe_layer_cached(moe_expert_cache *c, const moe_dims *dims, const moe_weights *weights, const uint16_t *x,
                            const int32_t *token_ids, float *y, void *ws, void *stream) {
    if (!c || !dims || !weights) return MOE_ERR_INVALID_ARG;
    moe_dims d = c->dims;
    d.T = dims->T;
    if (memcmp(&d, dims, sizeof d) != 0) return MOE_ERR_INVALID_ARG;  // the cache's layer, any T
    size_t need = 0;
    moe_status st = moe_workspace_size(dims, &need);
    if (st != MOE_OK) return st;
    if (!ws || reinterpret_cast<uintptr_t>(ws) % 256) return MOE_ERR_INVALID_ARG;
    if (d.T == 0) return MOE_OK;
    if (!x || !y || reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(y) % 16)
        return MOE_ERR_INVALID_ARG;
    if (d.route == MOE_ROUTE_HASH && !token_ids) return MOE_ERR_INVALID_ARG;
    if (d.route == MOE_ROUTE_SOFTMAX_TOPK && !weights->w_router) return MOE_ERR_INVALID_ARG;
    if (d.d_ff_shared > 0 && (!weights->sw1 || !weights->sw3 || !weights->sw2)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const WsLayout L = ws_layout(d);
    uint8_t *w = static_cast<uint8_t *>(ws);
    int32_t *idx = reinterpret_cast<int32_t *>(w + L.topk_idx);
    float *gates = reinterpret_cast<float *>(w + L.topk_w);
    int32_t *counts = reinterpret_cast<int32_t *>(w + L.counts);
    int32_t *offsets = reinterpret_cast<int32_t *>(w + L.offsets);
    int32_t *perm = reinterpret_cast<int32_t *>(w + L.perm);
    int32_t *inv = reinterpret_cast<int32_t *>(w + L.inv_perm);
    int32_t *slot_of = reinterpret_cast<int32_t *>(w + L.slot_of);
    int32_t *idx_slot = reinterpret_cast<int32_t *>(w + L.idx_slot);
    float *rows = reinterpret_cast<float *>(w + L.out_rows);
    float *sh = d.d_ff_shared > 0 ? reinterpret_cast<float *>(w + L.sh_out) : nullptr;
    const int S = d.T * d.k;
    auto cuda = [](cudaError_t e) {
        if (e != cudaSuccess) fprintf(stderr, "libmoe: CUDA error: %s\n", cudaGetErrorString(e));
        return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
    };
    cudaError_t e;
    // 1. routing over all experts, then the ids to the host
    if ((e = launch_route(d, x, *weights, token_ids, idx, gates, reinterpret_cast<float *>(w + L.logits),
                          reinterpret_cast<float *>(w + L.rnorm), s)))
        return cuda(e);
    if (S > c->idx_cap) {
        cudaFreeHost(c->h_idx);
        c->h_idx = nullptr;
        c->idx_cap = 0;
        if ((e = cudaMallocHost(reinterpret_cast<void **>(&c->h_idx), (size_t)S * 4))) return cuda(e);
        c->idx_cap = S;
    }
    if ((e = cudaMemcpyAsync(c->h_idx, idx, (size_t)S * 4, cudaMemcpyDeviceToHost, s))) return cuda(e);
    if ((e = cudaStreamSynchronize(s))) return cuda(e);
    // 2. the experts this batch touches, cached ones first, in waves of `slots`
    std::vector<char> touched(d.E, 0);
    for (int i = 0; i < S; ++i) {
        const int ex = c->h_idx[i];
        if (ex >= 0 && ex < d.E) touched[ex] = 1;
        // an id outside [0, E) only comes with a device error already set (hash draw cap)
    }
    std::vector<int> order;
    for (int ex = 0; ex < d.E; ++ex)
        if (touched[ex] && c->expert_slot[ex] >= 0) order.push_back(ex);
    for (int ex = 0; ex < d.E; ++ex)
        if (touched[ex] && c->expert_slot[ex] < 0) order.push_back(ex);
    moe_dims dc = d;  // the layer over the slots
    dc.E = c->slots;
    moe_weights wc = *weights;
    wc.w1 = c->dev[0];
    wc.w3 = c->dev[1];
    wc.w2 = c->dev[2];
    const bool r16 = tc_path_applies(dc);
    const int nwave = order.empty() ? 1 : (int)((order.size() + c->slots - 1) / c->slots);
    for (int wv = 0; wv < nwave; ++wv) {
        const int b = wv * c->slots, n = std::min<int>(c->slots, (int)order.size() - b);
        ++c->tick;
        std::vector<char> keep(c->slots, 0);
        for (int i = 0; i < n; ++i) {
            const int sl = c->expert_slot[order[b + i]];
            if (sl >= 0) keep[sl] = 1;
        }
        for (int i = 0; i < n; ++i) {
            const int ex = order[b + i];
            int sl = c->expert_slot[ex];
            if (sl >= 0) {
                ++c->stats.hits;
            } else {  // least recently used slot this wave does not need
                int best = -1;
                for (int q = 0; q < c->slots; ++q)
                    if (!keep[q] && (best < 0 || c->last_use[q] < c->last_use[best])) best = q;
                sl = best;
                if (c->slot_expert[sl] >= 0) c->expert_slot[c->slot_expert[sl]] = -1;
                c->slot_expert[sl] = ex;
                c->expert_slot[ex] = sl;
                keep[sl] = 1;
                for (int m = 0; m < 3; ++m)
                    for (int p = 0; p < 3; ++p) {
                        const int64_t len = c->piece[m][p];
                        if ((e = cudaMemcpyAsync(c->dev[m] + c->dev_off[m][p] + (int64_t)sl * len,
                                                 c->host[m] + c->host_off[m][p] + (int64_t)ex * len, (size_t)len,
                                                 cudaMemcpyHostToDevice, s)))
                            return cuda(e);
                        c->stats.bytes_h2d += (uint64_t)len;
                    }
                ++c->stats.misses;
            }
            c->last_use[sl] = c->tick;
        }
        // 3. slot map of this wave, then permute / FFN / combine over the slots
        int32_t *map = c->h_map + (size_t)wv * d.E;  // one row per wave: the uploads may still be in flight
        for (int ex = 0; ex < d.E; ++ex) map[ex] = -1;
        for (int i = 0; i < n; ++i) map[order[b + i]] = c->expert_slot[order[b + i]];
        if ((e = cudaMemcpyAsync(slot_of, map, (size_t)d.E * 4, cudaMemcpyHostToDevice, s))) return cuda(e);
        cache_remap_kernel<<<(S + 255) / 256, 256, 0, s>>>(idx, S, d.E, slot_of, idx_slot);
        count_launches(1);
        if ((e = launch_permute(dc, idx_slot, counts, offsets, perm, inv, reinterpret_cast<int32_t *>(w + L.blkcnt),
                                reinterpret_cast<int32_t *>(w + L.blkbase), L.nblk, s, 0, true)))
            return cuda(e);
        float *shw = wv == 0 ? sh : nullptr;  // the shared expert once, in the first wave
        if ((e = launch_expert_ffn(dc, wc, x, offsets, perm, rows, shw, w, L, s, false, r16))) return cuda(e);
        if (r16)
            e = launch_combine_bf16(dc, reinterpret_cast<const uint16_t *>(rows), inv, gates, shw, y, s, wv > 0);
        else
            e = launch_combine(dc, rows, inv, gates, shw, y, s, false, wv > 0);
        if (e) return cuda(e);
        ++c->stats.waves;
    }
    ++c->stats.calls;
    return MOE_OK;
}

}  // extern "C"
