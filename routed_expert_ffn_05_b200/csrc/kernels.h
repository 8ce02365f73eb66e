// Internal launchers (host side), one per stage; all return cudaGetLastError().
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "layout.h"
#include "moe.h"

namespace moe {

constexpr int kHashMaxDraws = 1024;

// Device address of this device's error word (moe_get_device_error).
int *device_error_word();

// Host-side launch accounting (moe_debug_launch_count): every launcher adds
// the number of kernels it put on the stream.
void count_launches(int n);

// logits: [T][E] scratch; rnorm: [E] scratch (the tensor-core router).
cudaError_t launch_route(const moe_dims &d, const uint16_t *x, const moe_weights &w,
                         const int32_t *token_ids, int32_t *idx, float *gates, float *logits,
                         float *rnorm, cudaStream_t s);

// Batch router on the tensor cores (approximate logits, then the canonical
// logits of the candidates only), when it applies.
bool router_tc_applies(const moe_dims &d);
cudaError_t launch_router_approx(const moe_dims &d, const uint16_t *x, const moe_weights &w, float *approx,
                                 float *wnorm, cudaStream_t s);
cudaError_t launch_route_tc(const moe_dims &d, const uint16_t *x, const moe_weights &w, int32_t *idx, float *gates,
                            float *approx, float *wnorm, cudaStream_t s);

// Hash routing alone, with a caller-chosen draw cap (the layer uses kHashMaxDraws).
cudaError_t launch_hash_route(const moe_dims &d, const int32_t *token_ids, int max_draws, int32_t *idx, float *w,
                              cudaStream_t s);

// Histogram, scan and stable permutation over d.E experts whose ids start at
// ebase (0 for a whole layer); foreign_ok: ids outside [ebase, ebase + d.E)
// are dropped silently (the expert-parallel layer) instead of reported.
cudaError_t launch_permute(const moe_dims &d, const int32_t *idx, int32_t *counts, int32_t *offsets,
                           int32_t *perm, int32_t *inv_perm, int32_t *blkcnt, int32_t *blkbase,
                           int64_t nblk, cudaStream_t s, int ebase = 0, bool foreign_ok = false);

// `pdl`: launch programmatically after the preceding kernel (the decode FFN).
// `accumulate`: add the sum to y (no shared term) instead of writing it.
cudaError_t launch_combine(const moe_dims &d, const float *out_rows, const int32_t *inv_perm,
                           const float *gates, const float *shared, float *y, cudaStream_t s, bool pdl = false,
                           bool accumulate = false);
// The same with bf16 expert rows (the fused layer on the tensor-core path).
cudaError_t launch_combine_bf16(const moe_dims &d, const uint16_t *out_rows, const int32_t *inv_perm,
                                const float *gates, const float *shared, float *y, cudaStream_t s,
                                bool accumulate = false);

cudaError_t launch_quantize_weights(const moe_dims &d, int which, const float *w, uint8_t *canonical,
                                    cudaStream_t s);
cudaError_t launch_pack_weights(const moe_dims &d, int which, const uint8_t *canonical, uint8_t *packed,
                                cudaStream_t s);
cudaError_t launch_debug_dequant(const moe_dims &d, int which, const uint8_t *packed, int expert,
                                 float *out, cudaStream_t s);
// MX quantisation of activation rows: MXFP8 codes [rows][K], or MXFP4 (fp4)
// codes [rows][K/2]; E8M0 scales [rows][K/32].
cudaError_t launch_quant_act_bf16(const uint16_t *x, int64_t rows, int K, uint8_t *codes, uint8_t *scales,
                                  cudaStream_t s, bool fp4 = false);
cudaError_t launch_quant_act_f32(const float *x, int64_t rows, int K, uint8_t *codes, uint8_t *scales,
                                 cudaStream_t s, bool fp4 = false);

// Routed expert FFN over all permuted rows (ws gives h / h8 / x8 scratch), and
// the shared expert into `shared_out` when it is non-null.
// `prepared`: the fused decode routing kernel already ran on this workspace.
// `rows_bf16`: on the tensor-core path write the expert rows as bf16 (out_rows
// then points at T*k*d_model uint16 values); ignored by the other paths.
cudaError_t launch_expert_ffn(const moe_dims &d, const moe_weights &w, const uint16_t *x,
                              const int32_t *offsets, const int32_t *perm, float *out_rows,
                              float *shared_out, uint8_t *ws, const WsLayout &L, cudaStream_t s,
                              bool prepared = false, bool rows_bf16 = false);

// Decode-sized path (tensor-core GEMV over streamed weights), when it applies.
bool decode_path_applies(const moe_dims &d);
bool decode_route_applies(const moe_dims &d);
// Routes over all d.E experts; counts / offsets / perm / inv_perm cover the
// El experts from ebase (El < 0: all), the other slots get inv_perm -1.
cudaError_t launch_decode_route(const moe_dims &d, const uint16_t *x, const moe_weights &w, int32_t *idx,
                                float *gates, int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv_perm,
                                uint8_t *ws, const WsLayout &L, cudaStream_t s, int ebase = 0, int El = -1);
cudaError_t launch_decode_ffn(const moe_dims &d, const moe_weights &w, const uint16_t *x, const int32_t *offsets,
                              const int32_t *perm, float *out_rows, float *shared_out, uint8_t *ws,
                              const WsLayout &L, cudaStream_t s, bool prepared);

// Test hook of the decode FFN's inter-CTA wait (moe_debug_set_wait), on the
// current device: limit in ns (0 = the library's limit) and extra tiles to
// wait for that nobody publishes (0 = none).
cudaError_t set_debug_wait(uint64_t limit_ns, uint32_t extra);

// w4a8 with MXFP4 weights on the tensor cores (tcgen05 block-scaled MMA).
bool tc_path_applies(const moe_dims &d);
cudaError_t launch_tc_ffn(const moe_dims &d, const moe_weights &w, const uint16_t *x, const int32_t *offsets,
                          const int32_t *perm, float *out_rows, uint8_t *ws, const WsLayout &L, cudaStream_t s,
                          bool rows_bf16 = false);

// Token-tile plan (ustart [E+1]) and the slot -> row inverse of perm (row_of [S], -1 for slots without a row).
cudaError_t launch_tc_plan(const moe_dims &d, const int32_t *offsets, const int32_t *perm, int32_t *ustart,
                           int32_t *row_of, cudaStream_t s);

// w4a16 (bf16 activations, MXFP4 weights) on the tensor cores, batches the
// decode path does not take.
bool tc16_path_applies(const moe_dims &d);
cudaError_t launch_tc16_ffn(const moe_dims &d, const moe_weights &w, const uint16_t *x, const int32_t *offsets,
                            const int32_t *perm, float *out_rows, uint8_t *ws, const WsLayout &L, cudaStream_t s);

// The tensor-core path's activation staging alone (also a test hook).
cudaError_t launch_tc_gather(const moe_dims &d, const uint16_t *x, const int32_t *offsets, const int32_t *perm,
                             int32_t *ustart, int32_t *row_of, uint8_t *gx8, uint8_t *gxsf, cudaStream_t s);

cudaError_t launch_shared_ffn(const moe_dims &d, const moe_weights &w, const uint16_t *x, float *out,
                              float *hbuf, cudaStream_t s);

}  // namespace moe
