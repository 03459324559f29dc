// Launchers shared between the libtb translation units (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/tb.h"

namespace tb {

// ---- attention (attn.cu) ----
size_t attn_ws_bytes(const tb_dims &d);
int attn_splits(const tb_dims &d);
cudaError_t launch_attn(const tb_dims &d, const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                        const int32_t *ctx_len, int32_t sink, int32_t window,
                        const uint32_t *sel_bits, bool sparse, float scale, float *out, void *ws,
                        cudaStream_t st);

// ---- score + select (select.cu) ----
size_t select_ws_bytes(const tb_dims &d);
// group_reduce: -1 = one set per query head; 0 / 1 = one set per KV head from
// the largest / the fp32 sum of the group's head scores; 2 = one set per query
// head holding at most `budget` positions after neighbour fetch.
cudaError_t launch_score_select(const tb_dims &d, const float *qp, int64_t qp_stride,
                                const uint16_t *Kp, const int32_t *ctx_len, int32_t sink,
                                int32_t window, int32_t budget, int32_t nbr, int32_t group_reduce,
                                int32_t *idx, int32_t idx_cap, int32_t *count, uint32_t *sel_bits,
                                void *ws, cudaStream_t st);
cudaError_t launch_select_bits(const tb_dims &d, const int32_t *idx, int32_t idx_cap,
                               const int32_t *count, uint32_t *sel_bits, cudaStream_t st);

// ---- tensor-core GEMMs (gemm_tc.cu) ----
size_t predict_ws_bytes(int32_t batch, int32_t hidden, int32_t inter, int32_t n_out);
cudaError_t launch_project_keys(const tb_dims &d, const uint16_t *K, const uint16_t *Wk,
                                uint16_t *Kp, const int32_t *tok_begin, const int32_t *tok_count,
                                int32_t max_tok, void *ws, cudaStream_t st);
cudaError_t launch_predict_queries(const uint16_t *h, const uint16_t *W1, const uint16_t *W2,
                                   float *qp, int32_t batch, int32_t hidden, int32_t inter,
                                   int32_t n_out, void *ws, cudaStream_t st);

// ---- KV append (kv.cu) ----
cudaError_t launch_kv_append(const tb_dims &d, int32_t n_layers, const uint16_t *src, const uint64_t *caches,
                             const int32_t *ctx_len, void *ws, cudaStream_t st);

cudaError_t launch_bounded_wait_selftest(void *ws, long long budget_cycles, cudaStream_t st);

// Host error text for the calling thread (api.cu).
void set_error(const char *fmt, ...);

}  // namespace tb
