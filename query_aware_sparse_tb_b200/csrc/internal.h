// Launchers shared between the libtb translation units (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "../../include/tb.h"

namespace tb {

// ---- attention (attn.cu) ----
size_t attn_ws_bytes(const tb_dims &d);
int attn_splits(const tb_dims &d);
cudaError_t launch_attn(const tb_dims &d, const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                        const int32_t *ctx_len, int32_t sink, int32_t window,
                        const uint32_t *sel_bits, bool sparse, float scale, float *out, void *ws,
                        cudaStream_t st, float *part_out = nullptr, const int32_t *plan = nullptr);
cudaError_t launch_attn_plan(const tb_dims &d, const uint32_t *sel_bits, const int32_t *ctx_len, int32_t sink,
                             int32_t window, int32_t *plan, uint32_t *flags, cudaStream_t st);
cudaError_t launch_combine(const float *parts, int32_t n_parts, int32_t rows, int32_t head_dim, float *out,
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
// The one-kernel cluster path of launch_score_select (select_cluster.cu) for
// group_reduce -1, 0 and 1: whether it takes dims `d` (with one_wave: in one
// wave of clusters of long slices, where it beats the multi-kernel path), and
// the launch.
bool select_cluster_fits(const tb_dims &d, int32_t group_reduce, bool one_wave);
cudaError_t launch_score_select_cluster(const tb_dims &d, const float *qp, int64_t qp_stride, const uint16_t *Kp,
                                        const int32_t *ctx_len, int32_t sink, int32_t window, int32_t budget,
                                        int32_t nbr, int32_t group_reduce, int32_t *idx, int32_t idx_cap,
                                        int32_t *count, uint32_t *sel_bits, void *ws, cudaStream_t st);
// The scores of launch_score_select (group_reduce -1, 0, 1) as order-preserving
// keys in the workspace, nothing else (select.cu; the cluster path's first step).
cudaError_t launch_score_keys(const tb_dims &d, const float *qp, int64_t qp_stride, const uint16_t *Kp,
                              const int32_t *ctx_len, int32_t sink, int32_t window, int32_t group_reduce, void *ws,
                              cudaStream_t st);
cudaError_t launch_export_scores(const tb_dims &d, const void *ws, const int32_t *ctx_len, int32_t sink,
                                 int32_t window, float *scores, cudaStream_t st);
cudaError_t launch_export_candidates(const tb_dims &d, const void *ws, const int32_t *idx, int32_t idx_cap,
                                     const int32_t *count, int32_t budget, int32_t pos_offset, uint64_t *cand,
                                     cudaStream_t st);
cudaError_t launch_merge_candidates(const tb_dims &d, const uint64_t *cand, int32_t n_ranks, int32_t budget,
                                    const int32_t *ctx_len, int32_t sink, int32_t window, int32_t nbr, int32_t *idx,
                                    int32_t idx_cap, int32_t *count, int32_t shard_begin, int32_t shard_len,
                                    int32_t local_cap, uint32_t *local_bits, uint32_t *flags, cudaStream_t st);
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
// The calling thread's attention launch mode (tb_attn_set_launch_mode, api.cu).
int attn_launch_mode();
// The calling thread's selection algorithm (tb_select_set_algorithm, api.cu).
int select_algorithm();

// Host-side argument checks of the attention entry points (api.cu), shared by
// tb_sparse_decode_attn, tb_decode_attn and tb_sparse_decode_attn_noalloc so
// that all of them accept exactly the same dims and pointers.  `sel_bits`,
// `sink` and `window` are checked only when `sparse` is true.
tb_status check_attn_args(const char *fn, const tb_dims *dims, const uint16_t *Q, const uint16_t *K,
                          const uint16_t *V, const int32_t *ctx_len, float scale, float *out, bool sparse,
                          const uint32_t *sel_bits, int32_t sink, int32_t window);

// ---- per-device host state (api.cu) ----
// Kernel attributes (the dynamic shared-memory limit) and the SM count belong
// to a device, not to the process: a process may drive several GPUs.
constexpr int kMaxDevices = 64;
// Raise kernel `fn`'s dynamic shared-memory limit to at least `bytes` on the
// current device; `done` is the caller's per-kernel record [kMaxDevices] of
// the limit already set on each device.
cudaError_t ensure_dynamic_smem(const void *fn, int bytes, std::atomic<int> *done);
// Multiprocessors of the current device (148 when it cannot be queried).
int num_sms();

}  // namespace tb
