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

cudaError_t launch_route(const moe_dims &d, const uint16_t *x, const moe_weights &w,
                         const int32_t *token_ids, int32_t *idx, float *gates, float *logits,
                         cudaStream_t s);

cudaError_t launch_permute(const moe_dims &d, const int32_t *idx, int32_t *counts, int32_t *offsets,
                           int32_t *perm, int32_t *inv_perm, int32_t *blkcnt, int32_t *blkbase,
                           int64_t nblk, cudaStream_t s);

// `pdl`: launch programmatically after the preceding kernel (the decode FFN).
cudaError_t launch_combine(const moe_dims &d, const float *out_rows, const int32_t *inv_perm,
                           const float *gates, const float *shared, float *y, cudaStream_t s, bool pdl = false);
// The same with bf16 expert rows (the fused layer on the tensor-core path).
cudaError_t launch_combine_bf16(const moe_dims &d, const uint16_t *out_rows, const int32_t *inv_perm,
                                const float *gates, const float *shared, float *y, cudaStream_t s);

cudaError_t launch_quantize_weights(const moe_dims &d, int which, const float *w, uint8_t *canonical,
                                    cudaStream_t s);
cudaError_t launch_pack_weights(const moe_dims &d, int which, const uint8_t *canonical, uint8_t *packed,
                                cudaStream_t s);
cudaError_t launch_debug_dequant(const moe_dims &d, int which, const uint8_t *packed, int expert,
                                 float *out, cudaStream_t s);
cudaError_t launch_quant_act_bf16(const uint16_t *x, int64_t rows, int K, uint8_t *codes, uint8_t *scales,
                                  cudaStream_t s);
cudaError_t launch_quant_act_f32(const float *x, int64_t rows, int K, uint8_t *codes, uint8_t *scales,
                                 cudaStream_t s);

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
cudaError_t launch_decode_route(const moe_dims &d, const uint16_t *x, const moe_weights &w, int32_t *idx,
                                float *gates, int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv_perm,
                                uint8_t *ws, const WsLayout &L, cudaStream_t s);
cudaError_t launch_decode_ffn(const moe_dims &d, const moe_weights &w, const uint16_t *x, const int32_t *offsets,
                              const int32_t *perm, float *out_rows, float *shared_out, uint8_t *ws,
                              const WsLayout &L, cudaStream_t s, bool prepared);

// w4a8 with MXFP4 weights on the tensor cores (tcgen05 block-scaled MMA).
bool tc_path_applies(const moe_dims &d);
cudaError_t launch_tc_ffn(const moe_dims &d, const moe_weights &w, const uint16_t *x, const int32_t *offsets,
                          const int32_t *perm, float *out_rows, uint8_t *ws, const WsLayout &L, cudaStream_t s,
                          bool rows_bf16 = false);

cudaError_t launch_shared_ffn(const moe_dims &d, const moe_weights &w, const uint16_t *x, float *out,
                              float *hbuf, cudaStream_t s);

}  // namespace moe
