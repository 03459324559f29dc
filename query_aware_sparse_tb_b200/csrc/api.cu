// libtb C ABI: host-side validation and dispatch.  Every entry point checks its
// arguments before any CUDA call, so an invalid call returns an error without
// touching the device.  See include/tb.h for the contract of each call.
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace tb {

static thread_local char g_err[512] = "";
static thread_local int g_attn_mode = TB_ATTN_WAIT_ALL;
static thread_local int g_select_algo = TB_SELECT_AUTO;

int attn_launch_mode() { return g_attn_mode; }
int select_algorithm() { return g_select_algo; }
static std::mutex g_state_mu;  // serialises one-time per-device kernel set-up

void set_error(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
}

namespace {

constexpr int kMaxCtxSelect = 1 << 19;
constexpr int kMaxInclusiveBudget = 8192;
constexpr int kMaxCtxAttn = 1 << 22;

tb_status fail(tb_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return s;
}

bool aligned16(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// bf16 tensors are read with 16-byte vector loads, cp.async and TMA
#define TB_CHECK_PTR_IN(p, fn)                                                               \
    do {                                                                                     \
        if (!aligned16(p))                                                                   \
            return fail(TB_ERR_INVALID_ARG, "%s: pointer '%s' is null or not 16-byte aligned", \
                        fn, #p);                                                             \
    } while (0)
// int32 / float / uint32 arrays are accessed a word at a time
#define TB_CHECK_PTR4_IN(p, fn)                                                              \
    do {                                                                                     \
        if (!aligned4(p))                                                                    \
            return fail(TB_ERR_INVALID_ARG, "%s: pointer '%s' is null or not 4-byte aligned",  \
                        fn, #p);                                                             \
    } while (0)
#define TB_CHECK_PTR(p) TB_CHECK_PTR_IN(p, __func__)
#define TB_CHECK_PTR4(p) TB_CHECK_PTR4_IN(p, __func__)

tb_status check_dims(const tb_dims *d, bool need_dproj, const char *fn) {
    if (!d) return fail(TB_ERR_INVALID_ARG, "%s: dims is null", fn);
    if (d->batch < 1 || d->n_q_heads < 1 || d->n_kv_heads < 1 || d->ctx_cap < 1)
        return fail(TB_ERR_INVALID_ARG, "%s: batch, head counts and ctx_cap must be >= 1", fn);
    if (d->n_q_heads % d->n_kv_heads != 0)
        return fail(TB_ERR_INVALID_ARG, "%s: n_q_heads (%d) not a multiple of n_kv_heads (%d)", fn,
                    d->n_q_heads, d->n_kv_heads);
    // batch and KV heads index grid dimensions whose limit is 65535
    if (d->batch > 65535 || d->n_kv_heads > 65535)
        return fail(TB_ERR_UNSUPPORTED, "%s: batch (%d) and n_kv_heads (%d) must be <= 65535", fn, d->batch,
                    d->n_kv_heads);
    if (d->n_q_heads / d->n_kv_heads != 4)
        return fail(TB_ERR_UNSUPPORTED, "%s: only GQA groups of 4 query heads are built (got %d)", fn,
                    d->n_q_heads / d->n_kv_heads);
    if (d->head_dim != 64 && d->head_dim != 128)
        return fail(TB_ERR_UNSUPPORTED, "%s: head_dim %d not built (64, 128)", fn, d->head_dim);
    if (need_dproj && d->d_proj != 16 && d->d_proj != 32)
        return fail(TB_ERR_UNSUPPORTED, "%s: d_proj %d not built (16, 32)", fn, d->d_proj);
    return TB_OK;
}

tb_status check_ws(void *ws, size_t have, size_t need, const char *fn) {
    if (!aligned16(ws)) return fail(TB_ERR_INVALID_ARG, "%s: workspace is null or not 16-byte aligned", fn);
    if (have < need)
        return fail(TB_ERR_WORKSPACE, "%s: workspace has %zu bytes, needs %zu", fn, have, need);
    return TB_OK;
}

tb_status cuda_status(cudaError_t e, const char *fn) {
    if (e == cudaSuccess) return TB_OK;
    return fail(TB_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
}

}  // namespace

tb_status check_attn_args(const char *fn, const tb_dims *dims, const uint16_t *Q, const uint16_t *K,
                          const uint16_t *V, const int32_t *ctx_len, float scale, float *out, bool sparse,
                          const uint32_t *sel_bits, int32_t sink, int32_t window) {
    tb_status s;
    if ((s = check_dims(dims, false, fn)) != TB_OK) return s;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V))
        return fail(TB_ERR_INVALID_ARG, "%s: Q, K and V must be non-null and 16-byte aligned", fn);
    if (!aligned4(ctx_len) || !aligned4(out))
        return fail(TB_ERR_INVALID_ARG, "%s: ctx_len and out must be non-null and 4-byte aligned", fn);
    if (dims->ctx_cap > kMaxCtxAttn)
        return fail(TB_ERR_UNSUPPORTED, "%s: ctx_cap %d above %d", fn, dims->ctx_cap, kMaxCtxAttn);
    if (!isfinite(scale)) return fail(TB_ERR_INVALID_ARG, "%s: scale is not finite", fn);
    if (sparse) {
        if (!aligned4(sel_bits))
            return fail(TB_ERR_INVALID_ARG, "%s: pointer 'sel_bits' is null or not 4-byte aligned", fn);
        if (sink < 0 || window < 1) return fail(TB_ERR_INVALID_ARG, "%s: need sink >= 0 and window >= 1", fn);
    }
    return TB_OK;
}

cudaError_t ensure_dynamic_smem(const void *fn, int bytes, std::atomic<int> *done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::atomic<int> &have = done[dev];
    if (have.load(std::memory_order_acquire) >= bytes) return cudaSuccess;
    std::lock_guard<std::mutex> lock(g_state_mu);
    if (have.load(std::memory_order_relaxed) >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) have.store(bytes, std::memory_order_release);
    return e;
}

int num_sms() {
    static std::atomic<int> sms[kMaxDevices];  // zero-initialised (static storage)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    std::atomic<int> &have = sms[dev];
    int n = have.load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
        have.store(n, std::memory_order_relaxed);
    }
    return n;
}

}  // namespace tb

using namespace tb;

extern "C" {

int32_t tb_abi_version(void) { return TB_ABI_VERSION; }

const char *tb_status_str(tb_status s) {
    switch (s) {
        case TB_OK: return "TB_OK";
        case TB_ERR_INVALID_ARG: return "TB_ERR_INVALID_ARG";
        case TB_ERR_UNSUPPORTED: return "TB_ERR_UNSUPPORTED";
        case TB_ERR_CUDA: return "TB_ERR_CUDA";
        case TB_ERR_WORKSPACE: return "TB_ERR_WORKSPACE";
        case TB_ERR_DEVICE_FLAG: return "TB_ERR_DEVICE_FLAG";
    }
    return "TB_ERR_UNKNOWN";
}

const char *tb_last_error(void) { return g_err; }

tb_status tb_attn_set_launch_mode(int32_t mode) {
    if (mode != TB_ATTN_WAIT_ALL && mode != TB_ATTN_PREFETCH_KV)
        return fail(TB_ERR_INVALID_ARG, "tb_attn_set_launch_mode: unknown mode %d", mode);
    g_attn_mode = mode;
    return TB_OK;
}

int32_t tb_attn_launch_mode(void) { return g_attn_mode; }

tb_status tb_select_set_algorithm(int32_t algorithm) {
    if (algorithm != TB_SELECT_AUTO && algorithm != TB_SELECT_MULTI_KERNEL && algorithm != TB_SELECT_CLUSTER)
        return fail(TB_ERR_INVALID_ARG, "tb_select_set_algorithm: unknown algorithm %d", algorithm);
    g_select_algo = algorithm;
    return TB_OK;
}

int32_t tb_select_algorithm(void) { return g_select_algo; }

size_t tb_score_select_workspace_bytes(const tb_dims *dims) {
    if (check_dims(dims, true, __func__) != TB_OK || dims->ctx_cap > kMaxCtxSelect) return 0;
    return select_ws_bytes(*dims);
}

size_t tb_attn_workspace_bytes(const tb_dims *dims) {
    if (check_dims(dims, false, __func__) != TB_OK || dims->ctx_cap > kMaxCtxAttn) return 0;
    return attn_ws_bytes(*dims);
}

size_t tb_predict_queries_workspace_bytes(int32_t batch, int32_t hidden, int32_t inter, int32_t n_out) {
    if (batch < 1 || batch > 16 || hidden < 256 || hidden % 256 || inter < 256 || inter % 256 ||
        n_out < 128 || n_out % 128)
        return 0;
    return predict_ws_bytes(batch, hidden, inter, n_out);
}

size_t tb_project_keys_workspace_bytes(void) { return kWsHeaderBytes; }

tb_status tb_workspace_init(void *ws, size_t ws_bytes, void *stream) {
    if (!aligned16(ws) || ws_bytes < (size_t)kWsHeaderBytes)
        return fail(TB_ERR_INVALID_ARG, "tb_workspace_init: bad workspace");
    return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream), __func__);
}

tb_status tb_workspace_check(void *ws, size_t ws_bytes, uint32_t *flags, void *stream) {
    if (!aligned16(ws) || ws_bytes < (size_t)kWsHeaderBytes || !flags)
        return fail(TB_ERR_INVALID_ARG, "tb_workspace_check: bad arguments");
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t v = 0;
    tb_status s;
    // read and clear the word in the caller's stream order, so that a kernel
    // queued after this call can never have its flag cleared
    if ((s = cuda_status(cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, st), __func__)) != TB_OK) return s;
    if ((s = cuda_status(cudaMemsetAsync(ws, 0, 4, st), __func__)) != TB_OK) return s;
    if ((s = cuda_status(cudaStreamSynchronize(st), __func__)) != TB_OK) return s;
    *flags = v;
    return v ? fail(TB_ERR_DEVICE_FLAG, "device flags 0x%x", v) : TB_OK;
}

tb_status tb_project_keys(const tb_dims *dims, const tb_bf16 *K, const tb_bf16 *Wk, tb_bf16 *Kp,
                          const int32_t *tok_begin, const int32_t *tok_count, int32_t max_tok,
                          void *ws, size_t ws_bytes, void *stream) {
    tb_status s;
    if ((s = check_dims(dims, true, __func__)) != TB_OK) return s;
    TB_CHECK_PTR(K); TB_CHECK_PTR(Wk); TB_CHECK_PTR(Kp); TB_CHECK_PTR4(tok_begin); TB_CHECK_PTR4(tok_count);
    if ((s = check_ws(ws, ws_bytes, kWsHeaderBytes, __func__)) != TB_OK) return s;
    if (max_tok < 0) return fail(TB_ERR_INVALID_ARG, "tb_project_keys: max_tok < 0");
    if ((long long)dims->batch * dims->n_kv_heads * dims->ctx_cap > 0x7fffffffLL)
        return fail(TB_ERR_UNSUPPORTED, "tb_project_keys: more than 2^31 cache rows");
    if (max_tok == 0) return TB_OK;
    return cuda_status(launch_project_keys(*dims, K, Wk, Kp, tok_begin, tok_count, max_tok, ws,
                                           (cudaStream_t)stream),
                       __func__);
}

tb_status tb_predict_queries(const tb_bf16 *h, const tb_bf16 *W1, const tb_bf16 *W2, float *qp,
                             int32_t batch, int32_t hidden, int32_t inter, int32_t n_out, void *ws,
                             size_t ws_bytes, void *stream) {
    TB_CHECK_PTR(h); TB_CHECK_PTR(W1); TB_CHECK_PTR(W2); TB_CHECK_PTR4(qp);
    if (batch < 1 || batch > 16)
        return fail(TB_ERR_UNSUPPORTED, "tb_predict_queries: batch %d outside [1, 16]", batch);
    if (hidden < 256 || hidden % 256 || inter < 256 || inter % 256)
        return fail(TB_ERR_UNSUPPORTED, "tb_predict_queries: hidden and inter must be multiples of 256");
    if (n_out < 128 || n_out % 128)
        return fail(TB_ERR_UNSUPPORTED, "tb_predict_queries: n_out must be a multiple of 128");
    tb_status s;
    if ((s = check_ws(ws, ws_bytes, predict_ws_bytes(batch, hidden, inter, n_out), __func__)) != TB_OK)
        return s;
    return cuda_status(launch_predict_queries(h, W1, W2, qp, batch, hidden, inter, n_out, ws,
                                              (cudaStream_t)stream),
                       __func__);
}

static tb_status score_select_impl(const char *fn, const tb_dims *dims, const float *qp,
                                   int64_t qp_batch_stride, const tb_bf16 *Kp, const int32_t *ctx_len,
                                   int32_t sink, int32_t window, int32_t budget, int32_t nbr,
                                   int32_t group_reduce, int32_t *idx, int32_t idx_cap, int32_t *count,
                                   uint32_t *sel_bits, void *ws, size_t ws_bytes, void *stream) {
    tb_status s;
    if ((s = check_dims(dims, true, fn)) != TB_OK) return s;
    TB_CHECK_PTR4_IN(qp, fn); TB_CHECK_PTR_IN(Kp, fn); TB_CHECK_PTR4_IN(ctx_len, fn); TB_CHECK_PTR4_IN(idx, fn);
    TB_CHECK_PTR4_IN(count, fn); TB_CHECK_PTR4_IN(sel_bits, fn);
    if (dims->ctx_cap > kMaxCtxSelect)
        return fail(TB_ERR_UNSUPPORTED, "%s: ctx_cap %d above %d", fn, dims->ctx_cap, kMaxCtxSelect);
    if (qp_batch_stride < (int64_t)dims->n_q_heads * dims->d_proj)
        return fail(TB_ERR_INVALID_ARG, "%s: qp_batch_stride %lld smaller than Hq*d'", fn,
                    (long long)qp_batch_stride);
    if (sink < 0 || window < 1 || budget < 1)
        return fail(TB_ERR_INVALID_ARG, "%s: need sink >= 0, window >= 1, budget >= 1", fn);
    if (nbr < 0 || nbr > 16) return fail(TB_ERR_INVALID_ARG, "%s: nbr %d outside [0, 16]", fn, nbr);
    // group_reduce 2 is the budget-inclusive mode: |I| <= budget
    if (group_reduce == 2 && budget > kMaxInclusiveBudget)
        return fail(TB_ERR_UNSUPPORTED, "%s: budget %d above %d", fn, budget, kMaxInclusiveBudget);
    const long long need_cap = group_reduce == 2 ? (long long)budget : (long long)(2 * nbr + 1) * budget;
    const long long min_cap = need_cap < dims->ctx_cap ? need_cap : dims->ctx_cap;
    if (idx_cap < min_cap)
        return fail(TB_ERR_INVALID_ARG, "%s: idx_cap %d < %lld (the largest possible selection)", fn, idx_cap,
                    min_cap);
    if ((s = check_ws(ws, ws_bytes, select_ws_bytes(*dims), fn)) != TB_OK) return s;
    if (g_select_algo == TB_SELECT_CLUSTER && group_reduce != 2 && !select_cluster_fits(*dims, group_reduce, false))
        return fail(TB_ERR_UNSUPPORTED, "%s: ctx_cap %d does not fit the cluster selection kernel", fn,
                    dims->ctx_cap);
    return cuda_status(launch_score_select(*dims, qp, qp_batch_stride, Kp, ctx_len, sink, window, budget, nbr,
                                           group_reduce, idx, idx_cap, count, sel_bits, ws, (cudaStream_t)stream),
                       fn);
}

tb_status tb_score_select(const tb_dims *dims, const float *qp, int64_t qp_batch_stride,
                          const tb_bf16 *Kp, const int32_t *ctx_len, int32_t sink, int32_t window,
                          int32_t budget, int32_t nbr, int32_t *idx, int32_t idx_cap, int32_t *count,
                          uint32_t *sel_bits, void *ws, size_t ws_bytes, void *stream) {
    return score_select_impl(__func__, dims, qp, qp_batch_stride, Kp, ctx_len, sink, window, budget, nbr, -1,
                             idx, idx_cap, count, sel_bits, ws, ws_bytes, stream);
}

tb_status tb_score_select_group(const tb_dims *dims, const float *qp, int64_t qp_batch_stride,
                                const tb_bf16 *Kp, const int32_t *ctx_len, int32_t sink, int32_t window,
                                int32_t budget, int32_t nbr, int32_t reduce, int32_t *idx, int32_t idx_cap,
                                int32_t *count, uint32_t *sel_bits, void *ws, size_t ws_bytes,
                                void *stream) {
    if (reduce != TB_GROUP_MAX && reduce != TB_GROUP_SUM)
        return fail(TB_ERR_INVALID_ARG, "%s: reduce %d is neither TB_GROUP_MAX nor TB_GROUP_SUM", __func__, reduce);
    return score_select_impl(__func__, dims, qp, qp_batch_stride, Kp, ctx_len, sink, window, budget, nbr, reduce,
                             idx, idx_cap, count, sel_bits, ws, ws_bytes, stream);
}

tb_status tb_kv_append(const tb_dims *dims, int32_t n_layers, const tb_bf16 *src, const uint64_t *caches,
                       const int32_t *ctx_len, void *ws, size_t ws_bytes, void *stream) {
    tb_status s;
    if ((s = check_dims(dims, false, __func__)) != TB_OK) return s;
    TB_CHECK_PTR(src); TB_CHECK_PTR4(ctx_len);
    if (!caches || (reinterpret_cast<uintptr_t>(caches) & 7u) != 0)
        return fail(TB_ERR_INVALID_ARG, "%s: caches is null or not 8-byte aligned", __func__);
    if (n_layers < 1 || (long long)n_layers * 2 * dims->batch * dims->n_kv_heads > (1LL << 30))
        return fail(TB_ERR_INVALID_ARG, "%s: n_layers %d out of range", __func__, n_layers);
    if ((s = check_ws(ws, ws_bytes, kWsHeaderBytes, __func__)) != TB_OK) return s;
    return cuda_status(launch_kv_append(*dims, n_layers, src, caches, ctx_len, ws, (cudaStream_t)stream), __func__);
}

tb_status tb_score_select_inclusive(const tb_dims *dims, const float *qp, int64_t qp_batch_stride,
                                    const tb_bf16 *Kp, const int32_t *ctx_len, int32_t sink, int32_t window,
                                    int32_t budget, int32_t nbr, int32_t *idx, int32_t idx_cap, int32_t *count,
                                    uint32_t *sel_bits, void *ws, size_t ws_bytes, void *stream) {
    return score_select_impl(__func__, dims, qp, qp_batch_stride, Kp, ctx_len, sink, window, budget, nbr, 2, idx,
                             idx_cap, count, sel_bits, ws, ws_bytes, stream);
}

tb_status tb_selftest_bounded_wait(void *ws, size_t ws_bytes, int64_t budget_cycles, void *stream) {
    tb_status s;
    if ((s = check_ws(ws, ws_bytes, kWsHeaderBytes, __func__)) != TB_OK) return s;
    if (budget_cycles < 1 || budget_cycles > 4000000000LL)
        return fail(TB_ERR_INVALID_ARG, "%s: budget_cycles %lld outside [1, 4e9]", __func__, (long long)budget_cycles);
    return cuda_status(launch_bounded_wait_selftest(ws, budget_cycles, (cudaStream_t)stream), __func__);
}

tb_status tb_score_select_scores(const tb_dims *dims, const void *ws, size_t ws_bytes, const int32_t *ctx_len,
                                 int32_t sink, int32_t window, float *scores, void *stream) {
    tb_status s;
    if ((s = check_dims(dims, true, __func__)) != TB_OK) return s;
    if (dims->ctx_cap > kMaxCtxSelect)
        return fail(TB_ERR_UNSUPPORTED, "%s: ctx_cap %d above %d", __func__, dims->ctx_cap, kMaxCtxSelect);
    TB_CHECK_PTR4(ctx_len); TB_CHECK_PTR4(scores);
    if (sink < 0 || window < 1) return fail(TB_ERR_INVALID_ARG, "%s: need sink >= 0 and window >= 1", __func__);
    if ((s = check_ws(const_cast<void *>(ws), ws_bytes, select_ws_bytes(*dims), __func__)) != TB_OK) return s;
    return cuda_status(launch_export_scores(*dims, ws, ctx_len, sink, window, scores, (cudaStream_t)stream),
                       __func__);
}

tb_status tb_select_export_candidates(const tb_dims *dims, const void *ws, size_t ws_bytes, const int32_t *idx,
                                      int32_t idx_cap, const int32_t *count, int32_t budget, int32_t pos_offset,
                                      uint64_t *cand, void *stream) {
    tb_status s;
    if ((s = check_dims(dims, true, __func__)) != TB_OK) return s;
    if (dims->ctx_cap > kMaxCtxSelect)
        return fail(TB_ERR_UNSUPPORTED, "%s: ctx_cap %d above %d", __func__, dims->ctx_cap, kMaxCtxSelect);
    TB_CHECK_PTR4(idx); TB_CHECK_PTR4(count);
    if (!cand || (reinterpret_cast<uintptr_t>(cand) & 7u) != 0)
        return fail(TB_ERR_INVALID_ARG, "%s: cand is null or not 8-byte aligned", __func__);
    if (idx_cap < 1 || budget < 1) return fail(TB_ERR_INVALID_ARG, "%s: need idx_cap >= 1 and budget >= 1", __func__);
    if (pos_offset < 0 || (long long)pos_offset + dims->ctx_cap > 0x7fffffffLL)
        return fail(TB_ERR_INVALID_ARG, "%s: pos_offset %d out of range", __func__, pos_offset);
    if ((s = check_ws(const_cast<void *>(ws), ws_bytes, select_ws_bytes(*dims), __func__)) != TB_OK) return s;
    return cuda_status(launch_export_candidates(*dims, ws, idx, idx_cap, count, budget, pos_offset, cand,
                                                (cudaStream_t)stream),
                       __func__);
}

tb_status tb_select_merge_candidates(const tb_dims *dims, const uint64_t *cand, int32_t n_ranks, int32_t budget,
                                     const int32_t *ctx_len, int32_t sink, int32_t window, int32_t nbr,
                                     int32_t *idx, int32_t idx_cap, int32_t *count, int32_t shard_begin,
                                     int32_t shard_len, int32_t local_cap, uint32_t *local_bits, void *ws,
                                     size_t ws_bytes, void *stream) {
    tb_status s;
    if ((s = check_dims(dims, true, __func__)) != TB_OK) return s;
    if (dims->ctx_cap > kMaxCtxSelect)
        return fail(TB_ERR_UNSUPPORTED, "%s: ctx_cap %d above %d", __func__, dims->ctx_cap, kMaxCtxSelect);
    if (!cand || (reinterpret_cast<uintptr_t>(cand) & 7u) != 0)
        return fail(TB_ERR_INVALID_ARG, "%s: cand is null or not 8-byte aligned", __func__);
    TB_CHECK_PTR4(ctx_len); TB_CHECK_PTR4(idx); TB_CHECK_PTR4(count); TB_CHECK_PTR4(local_bits);
    if (n_ranks < 1 || budget < 1 || (long long)n_ranks * budget > (1LL << 24))
        return fail(TB_ERR_INVALID_ARG, "%s: need n_ranks >= 1, budget >= 1, n_ranks*budget <= 2^24", __func__);
    if (sink < 0 || window < 1 || nbr < 0 || nbr > 16)
        return fail(TB_ERR_INVALID_ARG, "%s: need sink >= 0, window >= 1, 0 <= nbr <= 16", __func__);
    const long long need_cap = (long long)(2 * nbr + 1) * budget;
    if (idx_cap < (need_cap < dims->ctx_cap ? need_cap : dims->ctx_cap))
        return fail(TB_ERR_INVALID_ARG, "%s: idx_cap %d smaller than the largest possible selection", __func__, idx_cap);
    if (shard_begin < 0 || shard_begin % 32 != 0 || shard_len < 0 || local_cap < 1 || local_cap < shard_len ||
        (long long)shard_begin + shard_len > dims->ctx_cap)
        return fail(TB_ERR_INVALID_ARG, "%s: need 0 <= shard_begin (a multiple of 32), 0 <= shard_len <= local_cap, "
                    "and the shard inside ctx_cap", __func__);
    if ((s = check_ws(ws, ws_bytes, kWsHeaderBytes, __func__)) != TB_OK) return s;
    return cuda_status(launch_merge_candidates(*dims, cand, n_ranks, budget, ctx_len, sink, window, nbr, idx, idx_cap,
                                               count, shard_begin, shard_len, local_cap, local_bits,
                                               static_cast<uint32_t *>(ws), (cudaStream_t)stream),
                       __func__);
}

tb_status tb_sparse_decode_attn_partial(const tb_dims *dims, const tb_bf16 *Q, const tb_bf16 *K, const tb_bf16 *V,
                                        const int32_t *rows, const uint32_t *bits, float scale, float *part,
                                        void *ws, size_t ws_bytes, void *stream) {
    tb_status s = check_attn_args(__func__, dims, Q, K, V, rows, scale, part, true, bits, 0, 1);
    if (s != TB_OK) return s;
    if ((s = check_ws(ws, ws_bytes, attn_ws_bytes(*dims), __func__)) != TB_OK) return s;
    // sink 0 and window 0: no row is kept unless its bit is set
    return cuda_status(launch_attn(*dims, Q, K, V, rows, 0, 0, bits, true, scale, nullptr, ws, (cudaStream_t)stream,
                                   part),
                       __func__);
}

tb_status tb_attn_combine(const float *parts, int32_t n_parts, int32_t batch, int32_t n_q_heads, int32_t head_dim,
                          float *out, void *stream) {
    TB_CHECK_PTR4(parts); TB_CHECK_PTR4(out);
    if (n_parts < 1 || batch < 1 || n_q_heads < 1 || (long long)batch * n_q_heads > 0x7fffffffLL)
        return fail(TB_ERR_INVALID_ARG, "%s: need n_parts, batch and n_q_heads >= 1", __func__);
    if (head_dim != 64 && head_dim != 128)
        return fail(TB_ERR_UNSUPPORTED, "%s: head_dim %d not built (64, 128)", __func__, head_dim);
    return cuda_status(launch_combine(parts, n_parts, batch * n_q_heads, head_dim, out, (cudaStream_t)stream),
                       __func__);
}

tb_status tb_select_bits_from_idx(const tb_dims *dims, const int32_t *idx, int32_t idx_cap,
                                  const int32_t *count, uint32_t *sel_bits, void *stream) {
    tb_status s;
    if ((s = check_dims(dims, false, __func__)) != TB_OK) return s;
    TB_CHECK_PTR4(idx); TB_CHECK_PTR4(count); TB_CHECK_PTR4(sel_bits);
    if (idx_cap < 1) return fail(TB_ERR_INVALID_ARG, "tb_select_bits_from_idx: idx_cap < 1");
    if (dims->ctx_cap > kMaxCtxSelect)
        return fail(TB_ERR_UNSUPPORTED, "tb_select_bits_from_idx: ctx_cap above %d", kMaxCtxSelect);
    return cuda_status(launch_select_bits(*dims, idx, idx_cap, count, sel_bits, (cudaStream_t)stream), __func__);
}

tb_status tb_sparse_decode_attn(const tb_dims *dims, const tb_bf16 *Q, const tb_bf16 *K, const tb_bf16 *V,
                                const int32_t *ctx_len, int32_t sink, int32_t window,
                                const uint32_t *sel_bits, float scale, float *out, void *ws,
                                size_t ws_bytes, void *stream) {
    tb_status s = check_attn_args(__func__, dims, Q, K, V, ctx_len, scale, out, true, sel_bits, sink, window);
    if (s != TB_OK) return s;
    if ((s = check_ws(ws, ws_bytes, attn_ws_bytes(*dims), __func__)) != TB_OK) return s;
    return cuda_status(launch_attn(*dims, Q, K, V, ctx_len, sink, window, sel_bits, true, scale, out, ws,
                                   (cudaStream_t)stream),
                       __func__);
}

tb_status tb_sparse_decode_attn_planned(const tb_dims *dims, const tb_bf16 *Q, const tb_bf16 *K, const tb_bf16 *V,
                                        const int32_t *ctx_len, int32_t sink, int32_t window,
                                        const uint32_t *sel_bits, const int32_t *plan, float scale, float *out,
                                        void *ws, size_t ws_bytes, void *stream) {
    tb_status s = check_attn_args(__func__, dims, Q, K, V, ctx_len, scale, out, true, sel_bits, sink, window);
    if (s != TB_OK) return s;
    TB_CHECK_PTR4(plan);
    if ((s = check_ws(ws, ws_bytes, attn_ws_bytes(*dims), __func__)) != TB_OK) return s;
    return cuda_status(launch_attn(*dims, Q, K, V, ctx_len, sink, window, sel_bits, true, scale, out, ws,
                                   (cudaStream_t)stream, nullptr, plan),
                       __func__);
}

tb_status tb_attn_plan(const tb_dims *dims, const uint32_t *sel_bits, const int32_t *ctx_len, int32_t sink,
                       int32_t window, int32_t *plan, void *ws, size_t ws_bytes, void *stream) {
    tb_status s;
    if ((s = check_dims(dims, false, __func__)) != TB_OK) return s;
    if (dims->ctx_cap > kMaxCtxAttn)
        return fail(TB_ERR_UNSUPPORTED, "%s: ctx_cap %d above %d", __func__, dims->ctx_cap, kMaxCtxAttn);
    TB_CHECK_PTR4(sel_bits);
    TB_CHECK_PTR4(ctx_len);
    TB_CHECK_PTR4(plan);
    if (sink < 0 || window < 1) return fail(TB_ERR_INVALID_ARG, "%s: need sink >= 0 and window >= 1", __func__);
    if ((s = check_ws(ws, ws_bytes, kWsHeaderBytes, __func__)) != TB_OK) return s;
    return cuda_status(launch_attn_plan(*dims, sel_bits, ctx_len, sink, window, plan,
                                        static_cast<uint32_t *>(ws), (cudaStream_t)stream),
                       __func__);
}

tb_status tb_decode_attn(const tb_dims *dims, const tb_bf16 *Q, const tb_bf16 *K, const tb_bf16 *V,
                         const int32_t *ctx_len, float scale, float *out, void *ws, size_t ws_bytes,
                         void *stream) {
    tb_status s = check_attn_args(__func__, dims, Q, K, V, ctx_len, scale, out, false, nullptr, 0, 1);
    if (s != TB_OK) return s;
    if ((s = check_ws(ws, ws_bytes, attn_ws_bytes(*dims), __func__)) != TB_OK) return s;
    return cuda_status(launch_attn(*dims, Q, K, V, ctx_len, 0, 1, nullptr, false, scale, out, ws,
                                   (cudaStream_t)stream),
                       __func__);
}

}  // extern "C"
