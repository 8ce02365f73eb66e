// C ABI entry points (moe.h): host-side argument checks, workspace carving,
// kernel launches. Nothing here allocates device memory.
#include <stdio.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace moe {

__device__ int g_device_error = 0;

// Looked up once per device and kept for the life of the process (a
// cudaDeviceReset would invalidate it; the library is not meant to outlive one).
int *device_error_word() {
    static std::atomic<int *> addr[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    int *p = addr[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(reinterpret_cast<void **>(&p), g_device_error) != cudaSuccess) return nullptr;
        addr[dev].store(p, std::memory_order_release);
    }
    return p;
}

static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

static cudaEvent_t g_ffn_before = nullptr, g_ffn_after = nullptr;

// Routed-expert FFN bracketed by the optional profiling events.
static cudaError_t expert_ffn_timed(const moe_dims &d, const moe_weights &w, const uint16_t *x,
                                    const int32_t *offsets, const int32_t *perm, float *rows, float *shared,
                                    uint8_t *ws, const WsLayout &L, cudaStream_t s, bool prepared = false,
                                    bool rows_bf16 = false) {
    cudaError_t e;
    if (g_ffn_before && g_ffn_after && (e = cudaEventRecord(g_ffn_before, s)) != cudaSuccess) return e;
    if ((e = launch_expert_ffn(d, w, x, offsets, perm, rows, shared, ws, L, s, prepared, rows_bf16)) != cudaSuccess)
        return e;
    if (g_ffn_before && g_ffn_after) return cudaEventRecord(g_ffn_after, s);
    return cudaSuccess;
}

static bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static moe_status check_dims(const moe_dims *d) {
    if (!d) return MOE_ERR_INVALID_ARG;
    if (d->T < 0 || d->d_model <= 0 || d->d_ff <= 0 || d->E <= 0 || d->k <= 0) return MOE_ERR_INVALID_ARG;
    if (d->d_model % 256 || d->d_ff % 256) return MOE_ERR_INVALID_ARG;
    if (d->E > 1024 || d->k > 32 || d->k > d->E) return MOE_ERR_INVALID_ARG;
    if ((int64_t)d->T * d->k >= ((int64_t)1 << 31)) return MOE_ERR_INVALID_ARG;
    if (d->route != MOE_ROUTE_SOFTMAX_TOPK && d->route != MOE_ROUTE_HASH) return MOE_ERR_INVALID_ARG;
    if (d->act != MOE_A_BF16 && d->act != MOE_A_MXFP8 && d->act != MOE_A_MXFP4) return MOE_ERR_INVALID_ARG;
    if (d->wfmt != MOE_W_MXFP4 && d->wfmt != MOE_W_Q2K) return MOE_ERR_INVALID_ARG;
    if (d->d_ff_shared < 0 || d->d_ff_shared % 256) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

static bool valid_which(int32_t which) { return which == MOE_MAT_W1 || which == MOE_MAT_W2 || which == MOE_MAT_W3; }

static moe_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return MOE_OK;
    fprintf(stderr, "libmoe: CUDA error: %s\n", cudaGetErrorString(e));
    return MOE_ERR_CUDA;
}

static moe_status check_ws(const moe_dims *d, const void *ws) {
    if (!ws || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
    (void)d;
    return MOE_OK;
}

static moe_status check_weights(const moe_dims *d, const moe_weights *w, bool routed, bool router,
                                bool shared) {
    if (!w) return MOE_ERR_INVALID_ARG;
    if (routed && (!w->w1 || !w->w3 || !w->w2 || !aligned(w->w1, 256) || !aligned(w->w3, 256) ||
                   !aligned(w->w2, 256)))
        return MOE_ERR_INVALID_ARG;
    if (router && d->route == MOE_ROUTE_SOFTMAX_TOPK && (!w->w_router || !aligned(w->w_router, 16)))
        return MOE_ERR_INVALID_ARG;
    if (shared && d->d_ff_shared > 0 &&
        (!w->sw1 || !w->sw3 || !w->sw2 || !aligned(w->sw1, 16) || !aligned(w->sw3, 16) || !aligned(w->sw2, 16)))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

const char *moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported combination";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_DEVICE: return "device error word set";
        case MOE_ERR_TIMEOUT: return "bounded device wait gave up";
    }
    return "unknown status";
}

moe_status moe_workspace_size(const moe_dims *dims, size_t *bytes) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if (!bytes) return MOE_ERR_INVALID_ARG;
    *bytes = (size_t)ws_layout(*dims).total;
    return MOE_OK;
}

moe_status moe_packed_size(const moe_dims *dims, int32_t which, size_t *bytes) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if (!bytes || !valid_which(which)) return MOE_ERR_INVALID_ARG;
    *bytes = (size_t)(dims->wfmt == MOE_W_Q2K ? q2k_layout(*dims, which).total : mxfp4_layout(*dims, which).total);
    return MOE_OK;
}

moe_status moe_quantize_weights(const moe_dims *dims, int32_t which, const float *w, void *canonical,
                                void *stream) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if (!valid_which(which) || !w || !canonical || !aligned(w, 16) || !aligned(canonical, 256))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_quantize_weights(*dims, which, w, static_cast<uint8_t *>(canonical),
                                               static_cast<cudaStream_t>(stream)));
}

moe_status moe_pack_weights(const moe_dims *dims, int32_t which, const void *canonical, void *packed,
                            void *stream) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if (!valid_which(which) || !canonical || !packed || !aligned(canonical, 256) || !aligned(packed, 256))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_pack_weights(*dims, which, static_cast<const uint8_t *>(canonical),
                                           static_cast<uint8_t *>(packed), static_cast<cudaStream_t>(stream)));
}

moe_status moe_route(const moe_dims *dims, const uint16_t *x, const moe_weights *weights,
                     const int32_t *token_ids, int32_t *topk_idx, float *topk_w, void *ws, void *stream) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if ((st = check_weights(dims, weights, false, true, false)) != MOE_OK) return st;
    if ((st = check_ws(dims, ws)) != MOE_OK) return st;
    if (dims->T > 0 && (!topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
    if (dims->T > 0 && dims->route == MOE_ROUTE_HASH && !token_ids) return MOE_ERR_INVALID_ARG;
    if (dims->T > 0 && dims->route == MOE_ROUTE_SOFTMAX_TOPK && (!x || !aligned(x, 16))) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(*dims);
    float *logits = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + L.logits);
    float *rnorm = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + L.rnorm);
    return cuda_status(launch_route(*dims, x, *weights, token_ids, topk_idx, topk_w, logits, rnorm,
                                    static_cast<cudaStream_t>(stream)));
}

moe_status moe_permute(const moe_dims *dims, const int32_t *topk_idx, int32_t *counts, int32_t *offsets,
                       int32_t *perm, int32_t *inv_perm, void *ws, void *stream) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if ((st = check_ws(dims, ws)) != MOE_OK) return st;
    if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
    if (dims->T > 0 && (!topk_idx || !perm || !inv_perm)) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(*dims);
    uint8_t *w = static_cast<uint8_t *>(ws);
    return cuda_status(launch_permute(*dims, topk_idx, counts, offsets, perm, inv_perm,
                                      reinterpret_cast<int32_t *>(w + L.blkcnt),
                                      reinterpret_cast<int32_t *>(w + L.blkbase), L.nblk,
                                      static_cast<cudaStream_t>(stream)));
}

moe_status moe_expert_ffn(const moe_dims *dims, const moe_weights *weights, const uint16_t *x,
                          const int32_t *offsets, const int32_t *perm, float *out_rows, void *ws, void *stream) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if ((st = check_weights(dims, weights, true, false, false)) != MOE_OK) return st;
    if ((st = check_ws(dims, ws)) != MOE_OK) return st;
    if (dims->T > 0 && (!x || !offsets || !perm || !out_rows || !aligned(x, 16) || !aligned(out_rows, 16)))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(*dims);
    return cuda_status(expert_ffn_timed(*dims, *weights, x, offsets, perm, out_rows, nullptr,
                                        static_cast<uint8_t *>(ws), L, static_cast<cudaStream_t>(stream)));
}

moe_status moe_shared_ffn(const moe_dims *dims, const moe_weights *weights, const uint16_t *x, float *shared_out,
                          void *ws, void *stream) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if (dims->d_ff_shared == 0) return MOE_ERR_INVALID_ARG;
    if ((st = check_weights(dims, weights, false, false, true)) != MOE_OK) return st;
    if ((st = check_ws(dims, ws)) != MOE_OK) return st;
    if (dims->T > 0 && (!x || !shared_out || !aligned(x, 16) || !aligned(shared_out, 16))) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(*dims);
    float *hbuf = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + L.sh_h);
    return cuda_status(launch_shared_ffn(*dims, *weights, x, shared_out, hbuf, static_cast<cudaStream_t>(stream)));
}

moe_status moe_combine(const moe_dims *dims, const float *out_rows, const int32_t *inv_perm, const float *topk_w,
                       const float *shared_out, float *y, void *stream) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if (dims->T > 0 && (!out_rows || !inv_perm || !topk_w || !y || !aligned(out_rows, 16) || !aligned(y, 16) ||
                        (shared_out && !aligned(shared_out, 16))))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_combine(*dims, out_rows, inv_perm, topk_w, shared_out, y,
                                      static_cast<cudaStream_t>(stream)));
}

// The layer over the routed experts [ebase, ebase + El) of a layer of d.E
// (all of them for moe_layer), plus the shared expert when add_shared. Routing
// always runs over all d.E experts; the slots of experts outside the range
// take no row and add nothing to y. `w` holds the El experts' routed weights.
static moe_status layer_impl(const moe_dims &d, const moe_weights &wt, int ebase, int El, bool add_shared,
                             const uint16_t *x, const int32_t *token_ids, float *y, void *ws, cudaStream_t s) {
    const WsLayout L = ws_layout(d);  // the whole layer's layout covers every sub-range
    moe_dims dl = d;                  // the experts (and shared expert) this call computes
    dl.E = El;
    if (!add_shared) dl.d_ff_shared = 0;
    const bool part = El != d.E;
    uint8_t *w = static_cast<uint8_t *>(ws);
    int32_t *idx = reinterpret_cast<int32_t *>(w + L.topk_idx);
    float *gates = reinterpret_cast<float *>(w + L.topk_w);
    int32_t *counts = reinterpret_cast<int32_t *>(w + L.counts);
    int32_t *offsets = reinterpret_cast<int32_t *>(w + L.offsets);
    int32_t *perm = reinterpret_cast<int32_t *>(w + L.perm);
    int32_t *inv = reinterpret_cast<int32_t *>(w + L.inv_perm);
    float *rows = reinterpret_cast<float *>(w + L.out_rows);
    float *sh = dl.d_ff_shared > 0 ? reinterpret_cast<float *>(w + L.sh_out) : nullptr;
    cudaError_t e;
    const bool fused = decode_route_applies(d) && decode_path_applies(dl);
    if (fused) {
        if ((e = launch_decode_route(d, x, wt, idx, gates, counts, offsets, perm, inv, w, L, s, ebase, El)))
            return cuda_status(e);
    } else {
        if ((e = launch_route(d, x, wt, token_ids, idx, gates, reinterpret_cast<float *>(w + L.logits),
                              reinterpret_cast<float *>(w + L.rnorm), s)))
            return cuda_status(e);
        if ((e = launch_permute(dl, idx, counts, offsets, perm, inv, reinterpret_cast<int32_t *>(w + L.blkcnt),
                                reinterpret_cast<int32_t *>(w + L.blkbase), L.nblk, s, ebase, part)))
            return cuda_status(e);
    }
    // the tensor-core path hands its rows to the combine as bf16 (half the traffic)
    const bool r16 = tc_path_applies(dl);
    if ((e = expert_ffn_timed(dl, wt, x, offsets, perm, rows, sh, w, L, s, fused, r16))) return cuda_status(e);
    if (r16)
        return cuda_status(launch_combine_bf16(dl, reinterpret_cast<const uint16_t *>(rows), inv, gates, sh, y, s));
    return cuda_status(launch_combine(dl, rows, inv, gates, sh, y, s, decode_path_applies(dl)));
}

moe_status moe_layer(const moe_dims *dims, const moe_weights *weights, const uint16_t *x,
                     const int32_t *token_ids, float *y, void *ws, void *stream) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if ((st = check_weights(dims, weights, true, true, true)) != MOE_OK) return st;
    if ((st = check_ws(dims, ws)) != MOE_OK) return st;
    if (dims->T > 0 && (!x || !y || !aligned(x, 16) || !aligned(y, 16))) return MOE_ERR_INVALID_ARG;
    if (dims->T > 0 && dims->route == MOE_ROUTE_HASH && !token_ids) return MOE_ERR_INVALID_ARG;
    if (dims->T == 0) return MOE_OK;
    return layer_impl(*dims, *weights, 0, dims->E, true, x, token_ids, y, ws, static_cast<cudaStream_t>(stream));
}

moe_status moe_ep_range(int32_t E, int32_t rank, int32_t world, int32_t *begin, int32_t *end) {
    if (E <= 0 || world <= 0 || world > E || rank < 0 || rank >= world || !begin || !end) return MOE_ERR_INVALID_ARG;
    *begin = (int32_t)((int64_t)E * rank / world);
    *end = (int32_t)((int64_t)E * (rank + 1) / world);
    return MOE_OK;
}

moe_status moe_layer_ep(const moe_dims *dims, const moe_weights *weights, int32_t expert_begin, int32_t expert_end,
                        int32_t add_shared, const uint16_t *x, const int32_t *token_ids, float *y, void *ws,
                        void *stream) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if (expert_begin < 0 || expert_end <= expert_begin || expert_end > dims->E) return MOE_ERR_INVALID_ARG;
    moe_dims dw = *dims;  // the weights' own shape: expert_end - expert_begin routed experts
    dw.E = expert_end - expert_begin;
    if (!add_shared) dw.d_ff_shared = 0;
    if ((st = check_weights(&dw, weights, true, false, true)) != MOE_OK) return st;
    if ((st = check_weights(dims, weights, false, true, false)) != MOE_OK) return st;
    if ((st = check_ws(dims, ws)) != MOE_OK) return st;
    if (dims->T > 0 && (!x || !y || !aligned(x, 16) || !aligned(y, 16))) return MOE_ERR_INVALID_ARG;
    if (dims->T > 0 && dims->route == MOE_ROUTE_HASH && !token_ids) return MOE_ERR_INVALID_ARG;
    if (dims->T == 0) return MOE_OK;
    return layer_impl(*dims, *weights, expert_begin, expert_end - expert_begin, add_shared != 0, x, token_ids, y, ws,
                      static_cast<cudaStream_t>(stream));
}

moe_status moe_get_device_error(void *stream, int32_t *code) {
    if (!code) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t h = 0;
    const int32_t zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&h, g_device_error, sizeof h, 0, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_status(e);
    *code = h;
    return h ? MOE_ERR_DEVICE : MOE_OK;
}

moe_status moe_debug_dequant(const moe_dims *dims, int32_t which, const void *packed, int32_t expert, float *out,
                             void *stream) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if (!valid_which(which) || !packed || !out || expert < 0 || expert >= dims->E || !aligned(packed, 256))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_debug_dequant(*dims, which, static_cast<const uint8_t *>(packed), expert, out,
                                            static_cast<cudaStream_t>(stream)));
}

moe_status moe_debug_quant_act(const uint16_t *x, int32_t rows, int32_t K, uint8_t *codes, uint8_t *scales,
                               void *stream) {
    if (rows < 0 || K <= 0 || K % 32) return MOE_ERR_INVALID_ARG;
    if (rows > 0 && (!x || !codes || !scales || !aligned(codes, 16))) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_quant_act_bf16(x, rows, K, codes, scales, static_cast<cudaStream_t>(stream)));
}

moe_status moe_debug_hash_route(const moe_dims *dims, const int32_t *token_ids, int32_t max_draws, int32_t *topk_idx,
                                float *topk_w, void *stream) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if (dims->route != MOE_ROUTE_HASH || max_draws < 1 || max_draws > kHashMaxDraws) return MOE_ERR_INVALID_ARG;
    if (dims->T > 0 && (!token_ids || !topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_hash_route(*dims, token_ids, max_draws, topk_idx, topk_w, static_cast<cudaStream_t>(stream)));
}

moe_status moe_debug_tc_gather(const moe_dims *dims, const uint16_t *x, const int32_t *offsets, const int32_t *perm,
                               uint8_t *codes, uint8_t *atoms, int32_t *ustart, void *ws, void *stream) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if (!tc_path_applies(*dims)) return MOE_ERR_UNSUPPORTED;
    if ((st = check_ws(dims, ws)) != MOE_OK) return st;
    if (!x || !offsets || !perm || !codes || !atoms || !ustart || !aligned(x, 16) || !aligned(codes, 16))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(*dims);
    return cuda_status(launch_tc_gather(*dims, x, offsets, perm, ustart,
                                       reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + L.row_of), codes,
                                       atoms, static_cast<cudaStream_t>(stream)));
}

moe_status moe_debug_router_approx(const moe_dims *dims, const uint16_t *x, const moe_weights *weights,
                                  float *approx, float *wnorm, void *stream) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if ((st = check_weights(dims, weights, false, true, false)) != MOE_OK) return st;
    if (!router_tc_applies(*dims)) return MOE_ERR_UNSUPPORTED;
    if (!x || !approx || !wnorm || !aligned(x, 16)) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_router_approx(*dims, x, *weights, approx, wnorm, static_cast<cudaStream_t>(stream)));
}

moe_status moe_debug_set_wait(uint64_t limit_ns, uint32_t extra_tiles) {
    return cuda_status(set_debug_wait(limit_ns, extra_tiles));
}

uint64_t moe_debug_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

moe_status moe_debug_set_ffn_events(void *before, void *after) {
    if ((before == nullptr) != (after == nullptr)) return MOE_ERR_INVALID_ARG;
    g_ffn_before = static_cast<cudaEvent_t>(before);
    g_ffn_after = static_cast<cudaEvent_t>(after);
    return MOE_OK;
}

}  // extern "C"
