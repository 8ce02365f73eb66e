/*
 * moe.h — C ABI of the routed mixture-of-experts FFN layer over block-quantised
 * expert weights (libmoe.so, CUDA, sm_100a).
 *
 * The layer is the sparse MoE FFN of DeepSeek V4 Flash as the DwarfStar 4
 * pages describe it:
 *  - routed experts are quantised while the shared experts, projections and
 *    router stay unquantised ("DS4", dibi8.com, "Key architectural
 *    innovations" item 1; "DwarfStar", hysenlabs.com, "Model support and
 *    quantisation");
 *  - routed-expert weights are MXFP4 (the released FP4 weights kept as-is) or
 *    a 2-bit Q2_K-style format (hysenlabs.com, same section);
 *  - experts are picked by hashing or by a router ("DeepSeek V4 Flash ... on a
 *    Mac", grapeot.me, opening section: "hash MoE routing");
 *  - expert work is batched onto FP4 matrix instructions on Blackwell
 *    (hysenlabs.com, "Model support and quantisation").
 * Each expert is a SwiGLU FFN: h = silu(W1 a) * (W3 a), o = W2 h, with W1, W3
 * of shape [d_ff][d_model] and W2 of shape [d_model][d_ff]; quantisation
 * blocks run along the input dimension. The layer output is
 *     y[t] = sum_{j=0..k-1} w[t,j] * o_{e(t,j)}(x[t])  (+ shared expert (x[t])).
 *
 * Conventions for every entry point:
 *  - Pointers are DEVICE pointers unless stated otherwise; the caller owns and
 *    allocates every buffer. Scratch comes from the caller's workspace `ws`
 *    (size from moe_workspace_size, 256-byte aligned); the library allocates
 *    no device memory and keeps no per-call state.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream). Arguments are checked on the host first: a bad argument returns
 *    MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED and launches nothing.
 *  - Errors found by a kernel (an expert index outside [0, E), hash routing
 *    that needs more than 1024 draws for one token, a bounded wait that gave
 *    up, a perm that is not a permutation of the T*k slots) set a per-device
 *    error word; the outputs of that call are then
 *    undefined. Read and clear it with moe_get_device_error.
 *  - bf16 values travel as uint16_t bit patterns. Row-major everywhere.
 *  - Calls on distinct workspaces may run concurrently (on different streams,
 *    or beside other work that holds SMs: no kernel relies on all of its
 *    CTAs being resident at once); weights are read-only.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null pointer, bad size or shape, misaligned pointer */
    MOE_ERR_UNSUPPORTED = 2, /* a valid combination this build does not implement */
    MOE_ERR_CUDA = 3,        /* a CUDA runtime call failed (launch, copy, attribute) */
    MOE_ERR_DEVICE = 4,      /* the device error word was set (moe_get_device_error) */
    MOE_ERR_TIMEOUT = 5      /* a bounded device wait gave up */
} moe_status;

/* Routed-expert weight format. */
typedef enum { MOE_W_MXFP4 = 1, MOE_W_Q2K = 2 } moe_wfmt;
/* Activation mode of the routed experts: bf16 ("w4a16"), MXFP8 E4M3 with
 * per-32 E8M0 scales ("w4a8"), or MXFP4 E2M1 with per-32 E8M0 scales ("w4a4",
 * both GEMM operands on the FP4 matrix instructions that "DwarfStar",
 * hysenlabs.com, "Model support and quantisation", names for Blackwell). In
 * the quantised modes x and the hidden h are both quantised along their
 * length, by the rule the weights use (scale 2^(floor(log2 amax) - emax),
 * emax 8 for E4M3 and 2 for E2M1; elements round to nearest even and
 * saturate). */
typedef enum { MOE_A_BF16 = 0, MOE_A_MXFP8 = 1, MOE_A_MXFP4 = 2 } moe_amode;
/* Routing: top-k of bf16 router logits with softmax gates, or hash routing. */
typedef enum { MOE_ROUTE_SOFTMAX_TOPK = 0, MOE_ROUTE_HASH = 1 } moe_rmode;

/* Device error codes (moe_get_device_error). */
enum { MOE_DEVERR_NONE = 0, MOE_DEVERR_EXPERT_RANGE = 1, MOE_DEVERR_HASH_CAP = 2,
       MOE_DEVERR_TIMEOUT = 3, MOE_DEVERR_PERM = 4 };

/* Layer shape. Limits: d_model and d_ff multiples of 256 (of 32 for MXFP4),
 * 1 <= k <= min(E, 32), E <= 1024, T*k < 2^31. */
typedef struct {
    int32_t T;            /* tokens in this call (>= 0) */
    int32_t d_model;      /* d */
    int32_t d_ff;         /* F, routed expert hidden size */
    int32_t E;            /* routed experts */
    int32_t k;            /* experts per token */
    int32_t route;        /* moe_rmode */
    int32_t act;          /* moe_amode */
    int32_t wfmt;         /* moe_wfmt */
    int32_t d_ff_shared;  /* shared expert hidden size, 0 = no shared expert */
} moe_dims;

/* Weights of one layer (device pointers, read-only).
 *  w1, w3, w2: routed experts in the PACKED device layout written by
 *              moe_pack_weights (size from moe_packed_size);
 *  sw1, sw3:   shared expert bf16 [d_ff_shared][d_model], sw2 bf16
 *              [d_model][d_ff_shared], plain row-major; NULL when there is none;
 *  w_router:   router bf16 [E][d_model] (NULL for hash routing);
 *  router_bias: fp32 [E] added to the logits, or NULL. */
typedef struct {
    const void *w1, *w3, *w2;
    const uint16_t *sw1, *sw3, *sw2;
    const uint16_t *w_router;
    const float *router_bias;
} moe_weights;

/* Which routed-expert matrix: gate W1, up W3 ([E][d_ff][d_model]) or down W2
 * ([E][d_model][d_ff]). */
enum { MOE_MAT_W1 = 1, MOE_MAT_W3 = 3, MOE_MAT_W2 = 2 };

MOE_API const char *moe_status_string(moe_status s);

/* Bytes of workspace that moe_route .. moe_layer need for these dims (all
 * entry points share one workspace layout). Host only. No counterpart in the
 * pages: the caller owns all device memory. */
MOE_API moe_status moe_workspace_size(const moe_dims *dims, size_t *bytes);

/* ---- weights ------------------------------------------------------------
 * CANONICAL layout of one routed-expert matrix with N rows and K = input dim
 * (N = d_ff, K = d_model for W1/W3; N = d_model, K = d_ff for W2):
 *   MXFP4: codes u8 [E][N][K/2] (element 2i in the low nibble, OCP E2M1)
 *          followed by scales u8 [E][N][K/32] (E8M0) — E*N*K*17/32 bytes;
 *   Q2_K:  [E][N][K/256] super-blocks of 84 bytes: 16 bytes sc|m<<4,
 *          64 bytes of 2-bit quants (quant n at byte n/4, bits 2*(n%4)),
 *          fp16 d, fp16 dmin; w = d*sc*q - dmin*m.
 */

/* Quantise fp32 weights [E][N][K] (device) into the canonical layout
 * (device). MXFP4: per 32-block scale 2^(floor(log2 amax) - 2), elements
 * rounded to nearest-even E2M1 with saturation, all-zero block -> scale 127.
 * Q2_K: the min-max rule documented with the format. One-time, offline.
 * Formats: MXFP4 routed experts and the 2-bit Q2_K down projection
 * ("DwarfStar", hysenlabs.com, "Model support and quantisation"; "DS4",
 * dibi8.com, "Key architectural innovations" item 1). */
MOE_API moe_status moe_quantize_weights(const moe_dims *dims, int32_t which, const float *w,
                                void *canonical, void *stream);

/* Device bytes of one packed matrix (host only). */
MOE_API moe_status moe_packed_size(const moe_dims *dims, int32_t which, size_t *bytes);

/* Re-lay one canonical matrix (device) into the packed device layout used by
 * the kernels (device). One-time. `canonical` and `packed` must not overlap;
 * both 256-byte aligned. No counterpart in the pages (the pages keep the
 * released weights' format; this layout is this library's). */
MOE_API moe_status moe_pack_weights(const moe_dims *dims, int32_t which, const void *canonical,
                            void *packed, void *stream);

/* ---- the layer, stage by stage ---------------------------------------------
 * moe_route: picks k experts per token. The router is unquantised ("DS4",
 * dibi8.com, "Key architectural innovations" item 1); the model routes by
 * hashing ("DeepSeek V4 Flash ... on a Mac", grapeot.me, opening section).
 * Router logits are fp32 in one fixed order (32 contiguous chunks of d/32,
 * each a running fma from +0, then a balanced tree of adjacent pairs, then
 * the bias), so that expert choice is deterministic and reproducible.
 * topk_idx int32 [T][k], topk_w fp32 [T][k]; ties go to the lower expert index,
 * NaN logits last; gates are the softmax of the k chosen logits. Hash routing
 * (token_ids int32 [T], required): SplitMix64 seeded with the token id, expert =
 * output mod E, repeats skipped, gates 1/k. */
MOE_API moe_status moe_route(const moe_dims *dims, const uint16_t *x, const moe_weights *weights,
                     const int32_t *token_ids, int32_t *topk_idx, float *topk_w, void *ws,
                     void *stream);

/* Token-by-expert histogram, exclusive scan and stable permutation: the
 * grouping that batched expert work needs ("DwarfStar", hysenlabs.com, "Model
 * support and quantisation"). counts int32 [E], offsets int32 [E+1], perm
 * int32 [T*k] (row -> slot t*k+j, rows of one expert in ascending slot order),
 * inv_perm int32 [T*k] (slot -> row). Bit-exact and deterministic. A slot
 * whose expert index is outside [0, E) sets MOE_DEVERR_EXPERT_RANGE, takes no
 * row and gets inv_perm -1 (offsets[E] then counts only the valid slots). */
MOE_API moe_status moe_permute(const moe_dims *dims, const int32_t *topk_idx, int32_t *counts,
                       int32_t *offsets, int32_t *perm, int32_t *inv_perm, void *ws, void *stream);

/* Routed expert FFNs, batched per expert on quantised weights ("DwarfStar",
 * hysenlabs.com, "Model support and quantisation"; "DS4", dibi8.com, "Key
 * architectural innovations" item 1). For every permuted row: out_rows fp32
 * [T*k][d_model],
 * row r = o_{e}(x[perm[r] / k]) for the expert e whose segment holds r.
 * x bf16 [T][d_model]. The rows are offsets[E] <= T*k; perm[0 .. offsets[E])
 * holds distinct slots, as moe_permute writes it: a permutation of all T*k
 * slots when every slot has a valid expert (the MXFP8 path checks this:
 * MOE_DEVERR_PERM otherwise). In MXFP8 mode x and h are quantised on the
 * fly. */
MOE_API moe_status moe_expert_ffn(const moe_dims *dims, const moe_weights *weights, const uint16_t *x,
                          const int32_t *offsets, const int32_t *perm, float *out_rows, void *ws,
                          void *stream);

/* Shared expert, unquantised ("DS4", dibi8.com, "Key architectural
 * innovations" item 1): s fp32 [T][d_model] = W2s (bf16(silu(W1s x) *
 * (W3s x))), bf16 weights and activations, fp32 accumulation. */
MOE_API moe_status moe_shared_ffn(const moe_dims *dims, const moe_weights *weights, const uint16_t *x,
                          float *shared_out, void *ws, void *stream);

/* Gate-weighted combine of the routed experts' outputs (the MoE layer's sum,
 * "DeepSeek V4 Flash ... on a Mac", grapeot.me, opening section): y fp32
 * [T][d_model] = sum_{j ascending} topk_w[t][j] * out_rows[inv_perm[t*k+j]]
 * (+ shared_out[t]); slots with a negative inv_perm are skipped. shared_out
 * may be NULL. */
MOE_API moe_status moe_combine(const moe_dims *dims, const float *out_rows, const int32_t *inv_perm,
                       const float *topk_w, const float *shared_out, float *y, void *stream);

/* The whole layer, the routed MoE FFN over quantised experts ("DS4",
 * dibi8.com, "Key architectural innovations" item 1; "DwarfStar",
 * hysenlabs.com, "Model support and quantisation"): route -> permute ->
 * expert FFN (+ shared expert) -> combine, y fp32 [T][d_model]. token_ids is
 * required for hash routing and ignored otherwise. */
MOE_API moe_status moe_layer(const moe_dims *dims, const moe_weights *weights, const uint16_t *x,
                     const int32_t *token_ids, float *y, void *ws, void *stream);

/* ---- expert parallelism ------------------------------------------------------
 * The layer split across GPUs by routed expert, as the pages split it across
 * machines: each holds a contiguous share of the routed experts while the
 * router and the shared expert are replicated, and the partial sums are
 * exchanged ("DwarfStar", hysenlabs.com, "RDMA tensor parallelism and CUDA
 * tensor parallelism"). */

/* The contiguous expert range [*begin, *end) of rank `rank` of `world` for a
 * layer of E routed experts: begin = E rank / world, end = E (rank + 1) /
 * world (host only). Every expert belongs to exactly one rank. */
MOE_API moe_status moe_ep_range(int32_t E, int32_t rank, int32_t world, int32_t *begin, int32_t *end);

/* One rank's part of the layer: y fp32 [T][d_model] = the gate-weighted sum
 * over the slots whose expert lies in [expert_begin, expert_end), plus the
 * shared expert when add_shared (give it to one rank only). dims describe the
 * whole layer (E = all routed experts; the router covers all of them and the
 * routing is computed in full, identically on every rank). weights->w1, w3,
 * w2 hold only this rank's expert_end - expert_begin experts, packed for dims
 * with E = expert_end - expert_begin; sw1..sw2 may be NULL when !add_shared.
 * ws: a workspace for dims (moe_workspace_size). Summing y over ranks whose
 * ranges partition [0, E), exactly one with add_shared, gives moe_layer's y up
 * to the order of the fp32 sums. */
MOE_API moe_status moe_layer_ep(const moe_dims *dims, const moe_weights *weights, int32_t expert_begin,
                                int32_t expert_end, int32_t add_shared, const uint16_t *x, const int32_t *token_ids,
                                float *y, void *ws, void *stream);

/* ---- routed experts from host memory ---------------------------------------
 * The pages run models larger than memory by keeping the non-routed weights
 * resident and loading routed experts into a cache on a miss ("DwarfStar",
 * hysenlabs.com, "Running models larger than memory with SSD streaming";
 * baiwuji.top/articles/174, "Core features" item 2). Here every routed expert
 * lives in pinned host memory and `slots` of them at a time in HBM. */
typedef struct moe_expert_cache moe_expert_cache;

typedef struct {
    uint64_t calls;      /* moe_layer_cached calls */
    uint64_t waves;      /* expert waves run (a batch touching more experts than slots takes several) */
    uint64_t hits;       /* touched experts found in a slot */
    uint64_t misses;     /* touched experts copied in from host memory */
    uint64_t bytes_h2d;  /* bytes of expert weights copied host -> device */
} moe_cache_stats;

/* Creates a cache of `slots` (1 .. E) routed experts for the layer `dims`
 * (T ignored). host_w1, host_w3, host_w2: all E experts in the packed layout
 * (moe_pack_weights for dims, copied to host memory), PINNED host memory (page-
 * locked, e.g. cudaMallocHost), read-only and kept alive by the caller while
 * the cache lives. dev_w1, dev_w3, dev_w2: device buffers, 256-byte aligned,
 * of moe_packed_size for dims with E = slots; the cache owns their contents.
 * The cache object is host memory (plus small pinned staging buffers);
 * nothing on the device is allocated. Not thread-safe: one caller (one
 * stream) at a time. */
MOE_API moe_status moe_cache_create(const moe_dims *dims, int32_t slots, const void *host_w1, const void *host_w3,
                                    const void *host_w2, void *dev_w1, void *dev_w3, void *dev_w2,
                                    moe_expert_cache **cache);
MOE_API moe_status moe_cache_destroy(moe_expert_cache *cache);
MOE_API moe_status moe_cache_get_stats(const moe_expert_cache *cache, moe_cache_stats *stats);

/* moe_layer over the cache: same arguments and result as moe_layer for the
 * cache's layer (dims equal to the create dims except T); weights->w1, w3, w2
 * are ignored (the cache supplies the routed experts). The call routes on the
 * GPU, then SYNCHRONISES `stream` to read the expert choice on the host,
 * copies the missing experts in (least recently used slot first, one
 * cudaMemcpyAsync per contiguous piece), and runs the experts in waves of at
 * most `slots`: with one wave y is bit for bit moe_layer's staged-path result;
 * with several, the waves' sums are added in wave order. */
MOE_API moe_status moe_layer_cached(moe_expert_cache *cache, const moe_dims *dims, const moe_weights *weights,
                                    const uint16_t *x, const int32_t *token_ids, float *y, void *ws, void *stream);

/* Size of the scratch array built into the library for moe_layer_static_ws. */
#define MOE_STATIC_WS_BYTES (32u << 20)

/* moe_layer for callers that cannot allocate device memory. The pages have no
 * counterpart: this is a deployment convenience of this library.
 *
 * Who needs it: programs whose device memory belongs to another allocator (a
 * serving framework's pool, or an arena fixed at start-up, where one more
 * cudaMalloc would break the memory budget), latency-critical decode loops
 * that cannot pay for cudaMalloc / cudaFree (both may synchronise the device
 * and stall other streams), and deployments that forbid allocation after
 * initialisation. Instead of a caller workspace it uses one scratch array of
 * MOE_STATIC_WS_BYTES compiled into the library; every GPU that loads the
 * library holds that array until the process exits.
 *
 * Same arguments, results and errors as moe_layer minus `ws`. Returns
 * MOE_ERR_INVALID_ARG, launching nothing, when moe_workspace_size(dims) is
 * larger than MOE_STATIC_WS_BYTES (at d_model 4096, d_ff 2048, E 256, k 8
 * with a shared expert of d_ff 2048 that holds up to T = 97 tokens; a test
 * checks that bound against moe_workspace_size). It calls no cudaMalloc,
 * cudaFree or other allocating routine. The first call on a device looks up
 * the array's device address (cudaGetSymbolAddress, with that device
 * current) and keeps it for the life of the process (a cudaDeviceReset
 * invalidates it: do not reset a device and go on using the library); make
 * that first call before any stream capture. All calls on a device share the
 * one array and it keeps the previous call's contents (the layer writes or
 * clears every scratch byte before reading it), so calls whose execution
 * overlaps on the GPU race: serialise them, e.g. on one stream. */
MOE_API moe_status moe_layer_static_ws(const moe_dims *dims, const moe_weights *weights, const uint16_t *x,
                                       const int32_t *token_ids, float *y, void *stream);

/* Synchronises `stream`, returns the per-device error word in *code (host
 * pointer) and clears it. Returns MOE_ERR_DEVICE when it was set. */
MOE_API moe_status moe_get_device_error(void *stream, int32_t *code);

/* ---- test hooks ------------------------------------------------------------ */

/* Dequantise one matrix of one expert from the PACKED layout: out fp32 [N][K]
 * (device). Bit-exact decode of the format. */
MOE_API moe_status moe_debug_dequant(const moe_dims *dims, int32_t which, const void *packed,
                             int32_t expert, float *out, void *stream);

/* MXFP8-quantise bf16 rows: codes u8 [rows][K], scales u8 [rows][K/32]
 * (device), the same rule the layer applies to x. */
MOE_API moe_status moe_debug_quant_act(const uint16_t *x, int32_t rows, int32_t K, uint8_t *codes,
                               uint8_t *scales, void *stream);

/* Hash routing with a draw cap of max_draws (1 .. 1024; the layer uses 1024),
 * for tests of the cap: a token that needs more draws gets -1 in its unfilled
 * slots and sets MOE_DEVERR_HASH_CAP. dims->route must be MOE_ROUTE_HASH. */
MOE_API moe_status moe_debug_hash_route(const moe_dims *dims, const int32_t *token_ids, int32_t max_draws,
                                        int32_t *topk_idx, float *topk_w, void *stream);

/* The MXFP8 activation staging of the tensor-core path (MXFP4 weights, MXFP8
 * activations), alone, for byte-exact tests of what the GEMMs read: for the
 * permuted rows given by offsets / perm (as moe_permute writes them) it
 * writes codes u8 [T*k][d_model] (row r = the E4M3 codes of x[perm[r] / k]),
 * ustart int32 [E+1] (the first 128-row token tile of each expert) and the
 * E8M0 scale atoms u8 [ceil(T*k/128) + E][d_model/128][512]: the scale of
 * 32-block b of row r of expert e (r' = r - offsets[e]) is byte
 * (r' % 32) * 16 + ((r' % 128) / 32) * 4 + b % 4 of atom
 * (ustart[e] + r' / 128, b / 4). ws: a workspace for dims. */
MOE_API moe_status moe_debug_tc_gather(const moe_dims *dims, const uint16_t *x, const int32_t *offsets,
                                       const int32_t *perm, uint8_t *codes, uint8_t *atoms, int32_t *ustart,
                                       void *ws, void *stream);

/* The first step of the batch router (softmax routing, T >= 32), alone:
 * approximate logits approx fp32 [T][E] from one bf16 tensor-core GEMM (plus
 * the bias) and the router rows' 2-norms wnorm fp32 [E]. The router then
 * computes the canonical logit of every expert whose interval
 * [approx - B, approx + B] reaches the k-th largest lower bound, with
 * B = (d 2^-21 |x_t| wnorm[e] + 2^-20 (|approx| + |bias|) + 2^-100) (1 + 2^-8)
 * and |x_t| the fp32 2-norm of the token's row (both norms inflated by
 * 2^-8): tests check |approx - canonical| <= B. */
MOE_API moe_status moe_debug_router_approx(const moe_dims *dims, const uint16_t *x, const moe_weights *weights,
                                           float *approx, float *wnorm, void *stream);

/* Test hook of the decode path's one wait between CTAs (a down tile waiting
 * for its expert's gate/up tiles), on the current device, for tests of the
 * timeout path: give up after limit_ns instead of the library's 2 s, and wait
 * for extra_tiles more tiles than exist (a count nobody reaches). (0, 0)
 * restores the defaults. Synchronous; not for use while layers run. */
MOE_API moe_status moe_debug_set_wait(uint64_t limit_ns, uint32_t extra_tiles);

/* Number of kernels this library has launched in this process (host counter,
 * all devices and threads). For benchmarks that report their launch count. */
MOE_API uint64_t moe_debug_launch_count(void);

/* Profiling hook: when both are non-NULL, moe_layer and moe_expert_ffn record
 * `before` (a cudaEvent_t) on their stream right before the first routed-expert
 * FFN kernel and `after` right after the last one. NULL, NULL turns it off.
 * Process-wide; not for concurrent use from several threads. */
MOE_API moe_status moe_debug_set_ffn_events(void *before, void *after);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
