/*
 * tb.h — C ABI of the TokenButler decode-time selection and sparse-attention
 * library (libtb.so, CUDA kernels for sm_100a).
 *
 * The path (TokenButler technical summary, gist.science, sections
 * "Core architecture" (コアアーキテクチャ), "Inference strategy" (推論戦略) and
 * "Optimisations" (最適化)):
 *
 *   1. tb_project_keys       K' = K · W_kᵀ into d' dims, in batches of N tokens
 *   2. tb_predict_queries    producer-layer MLP: q' = SiLU(h·W1ᵀ)·W2ᵀ, G slots
 *   3+4. tb_score_select     s = q'·K'ᵀ over the candidates, top-B with
 *                            neighbour fetch outside the sink and window
 *   5. tb_sparse_decode_attn attention over sink ∪ window ∪ selected rows
 *   –  tb_decode_attn        dense decode attention (the comparator)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers are DEVICE pointers unless a comment says "host".  bf16 arrays
 *    (K, V, K', Q, W_k, W1, W2, h) and workspaces must be 16-byte aligned;
 *    int32, uint32 and float arrays 4-byte aligned.  No call allocates or
 *    frees device memory; the caller owns every buffer, including
 *    workspaces.  One exception holds memory: the fixed scratch of
 *    tb_sparse_decode_attn_noalloc (TB_NOALLOC_SCRATCH_BYTES = 4 MiB), a
 *    static device array that every GPU which loads libtb.so keeps until the
 *    process exits, whether or not that entry point is ever called.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call is
 *    asynchronous: it validates its arguments on the host, launches, and
 *    returns; it never synchronises the device.  The exceptions say so:
 *    tb_workspace_check synchronises its stream, and the first
 *    tb_sparse_decode_attn_noalloc call on a device waits for its set-up.
 *  - bf16 values are passed as raw 16-bit patterns (`tb_bf16`).
 *  - Caches use the layout [batch][n_kv_heads][ctx_cap][dim], row-contiguous
 *    per (sequence, KV head).  Query-head h belongs to KV head h / (Hq/Hkv).
 *  - Host-side argument errors return TB_ERR_INVALID_ARG or TB_ERR_UNSUPPORTED
 *    BEFORE any launch; the message is available from tb_last_error() on the
 *    calling thread.  A launch failure returns TB_ERR_CUDA.
 *  - Conditions only the device can see (a per-sequence context length outside
 *    [1, ctx_cap], a wait that timed out) never trap: the kernel clamps or
 *    skips, sets a bit in the workspace's flag word, and the caller reads it
 *    with tb_workspace_check().
 *  - Workspaces must be zeroed once before first use (tb_workspace_init); every
 *    call leaves its counters and histograms zeroed again.  Two calls that use
 *    the same workspace must not overlap on the device.
 */
#ifndef TB_H
#define TB_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TB_ABI_VERSION 10

typedef uint16_t tb_bf16;

typedef enum {
    TB_OK = 0,
    TB_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, bad shape */
    TB_ERR_UNSUPPORTED = 2,   /* valid but not built: head_dim, d', group size */
    TB_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed */
    TB_ERR_WORKSPACE = 4,     /* workspace too small */
    TB_ERR_DEVICE_FLAG = 5    /* tb_workspace_check found device-side flags */
} tb_status;

/* Device-side flag bits reported by tb_workspace_check(). */
#define TB_FLAG_CTX_RANGE   0x1u  /* some ctx_len[b] outside [1, ctx_cap]: clamped */
#define TB_FLAG_TIMEOUT     0x2u  /* a bounded wait gave up; the output is invalid */
#define TB_FLAG_IDX_OVERFLOW 0x4u /* selected set larger than idx_cap: truncated */
#define TB_FLAG_BAD_CACHE   0x8u  /* tb_kv_append: a cache address was null or misaligned: skipped */

/* Shapes shared by the cache-facing calls. */
typedef struct {
    int32_t batch;       /* sequences, <= 65535 */
    int32_t n_q_heads;   /* Hq  */
    int32_t n_kv_heads;  /* Hkv <= 65535; Hq / Hkv must be 4 */
    int32_t head_dim;    /* d:  64 or 128 */
    int32_t d_proj;      /* d': 16 or 32 */
    int32_t ctx_cap;     /* rows per (sequence, KV head) in K, V and K' */
} tb_dims;

int32_t     tb_abi_version(void);
const char *tb_status_str(tb_status s);
/* Message of the last non-OK status returned on this thread ("" if none). */
const char *tb_last_error(void);

/* ---- workspaces --------------------------------------------------------- */

/* Bytes of workspace each call needs (>= 256: the first 256 bytes hold the
 * device flag word).  0 is returned for invalid dims. */
size_t tb_score_select_workspace_bytes(const tb_dims *dims);
size_t tb_attn_workspace_bytes(const tb_dims *dims);           /* sparse and dense */
size_t tb_predict_queries_workspace_bytes(int32_t batch, int32_t hidden, int32_t inter,
                                          int32_t n_out);
size_t tb_project_keys_workspace_bytes(void);

/* Zero a workspace (cudaMemsetAsync).  Call once on a new workspace. */
tb_status tb_workspace_init(void *ws, size_t ws_bytes, void *stream);

/* Synchronise `stream`, copy the workspace's device flag word into *flags
 * (host), clear it, and return TB_ERR_DEVICE_FLAG if any bit was set. */
tb_status tb_workspace_check(void *ws, size_t ws_bytes, uint32_t *flags, void *stream);

/* ---- 1. key-cache projection -------------------------------------------- */
/* Each consumer layer projects its keys with a learned matrix into the d'
 * space of the predicted queries (summary, "Core architecture: key-cache
 * projection"); the projection runs once per batch of N new tokens rather than
 * at every step (summary, "Optimisations: batching").
 *
 *   Kp[b][g][t][:] = bf16_rne( sum_i K[b][g][t][i] * Wk[g][:][i] )   (fp32 accumulate)
 *
 * for t in [tok_begin[b], tok_begin[b] + tok_count[b]) ∩ [0, ctx_cap).
 *   K          [batch][Hkv][ctx_cap][d]   bf16
 *   Wk         [Hkv][d'][d]               bf16 (output-major: row j is output dim j)
 *   Kp         [batch][Hkv][ctx_cap][d']  bf16, only the rows above are written
 *   tok_begin  [batch] int32; a negative entry skips that sequence
 *   tok_count  [batch] int32
 *   max_tok    host: an upper bound on every tok_count[b] (sizes the grid)
 * Tensor cores (tcgen05) with TMA-loaded operands. */
tb_status tb_project_keys(const tb_dims *dims, const tb_bf16 *K, const tb_bf16 *Wk,
                          tb_bf16 *Kp, const int32_t *tok_begin, const int32_t *tok_count,
                          int32_t max_tok, void *ws, size_t ws_bytes, void *stream);

/* ---- 2. query prediction ------------------------------------------------- */
/* A light MLP takes the producer layer's hidden state and emits G
 * slot-specific low-dimensional queries per attention head (summary, "Core
 * architecture: query prediction").  Bias-free, SiLU between the products, the
 * activation rounded to bf16 before the second product:
 *
 *   a  = bf16_rne( SiLU( h · W1ᵀ ) )          fp32 accumulate
 *   qp = a · W2ᵀ                               fp32 accumulate and output
 *
 *   h   [batch][hidden] bf16;  W1 [inter][hidden] bf16;  W2 [n_out][inter] bf16
 *   qp  [batch][n_out] fp32, n_out = G * Hq * d', read as [batch][G][Hq][d']
 * batch <= 16; hidden, inter multiples of 256; n_out a multiple of 128.
 * Tensor cores (tcgen05), split-K over CTAs, deterministic reduction. */
tb_status tb_predict_queries(const tb_bf16 *h, const tb_bf16 *W1, const tb_bf16 *W2,
                             float *qp, int32_t batch, int32_t hidden, int32_t inter,
                             int32_t n_out, void *ws, size_t ws_bytes, void *stream);

/* ---- 3+4. scoring and budgeted selection ---------------------------------- */
/* Dot products of the predicted queries with the projected keys give cheap
 * importance scores for a dynamic per-token selection under a fixed budget
 * (summary, "Core architecture: scoring"); the first S tokens (sink) and the
 * last N (local window) are always kept and the importance buffer is filled
 * from the scores (summary, "Inference strategy"); the selected tokens are
 * expanded by their spatial neighbours (summary, "Optimisations: prediction
 * interval and neighbour fetch").  For each sequence b and query head h, with
 * T = ctx_len[b] and candidates C = [sink, T - window):
 *
 *   s[t]  = fp32( sum_j qp[b][h][j] * Kp[b][h/4][t][j] ),  t in C
 *   Top   = the `budget` members of C first in the order (s desc, t asc)
 *   I     = ( ∪_{t in Top} [t - nbr, t + nbr] ) ∩ C
 *
 *   qp         float [batch][..][Hq][d'] at qp + b*qp_batch_stride + h*d'
 *              (point at one slot of a [batch][G][Hq][d'] array; stride G*Hq*d')
 *   Kp         [batch][Hkv][ctx_cap][d'] bf16; rows of C must be projected
 *   ctx_len    [batch] int32 (device)
 *   idx        [batch][Hq][idx_cap] int32 out: I sorted ascending in
 *              idx[b][h][0 .. count[b][h]); the slots after those are not
 *              written
 *   count      [batch][Hq] int32 out: |I|
 *   sel_bits   [batch][Hq][ceil(ctx_cap/32)] uint32 out: bit t%32 of word t/32
 *              is 1 iff t in I (all other bits 0); this is what
 *              tb_sparse_decode_attn consumes
 *   idx_cap    >= min((2*nbr+1)*budget, ctx_cap)
 * Limits: budget >= 1, sink >= 0, window >= 1, 0 <= nbr <= 16, ctx_cap <= 524288.
 * The result is exact for the fp32 scores the kernel computes (radix select on
 * the order-preserving integer image of the scores, ties by position). */
tb_status tb_score_select(const tb_dims *dims, const float *qp, int64_t qp_batch_stride,
                          const tb_bf16 *Kp, const int32_t *ctx_len, int32_t sink,
                          int32_t window, int32_t budget, int32_t nbr, int32_t *idx,
                          int32_t idx_cap, int32_t *count, uint32_t *sel_bits, void *ws,
                          size_t ws_bytes, void *stream);

/* Group-shared variant (no counterpart on the pages; an alternative to their
 * per-attention-head selection for GQA).  The 4 query heads of a KV head
 * share one importance set, chosen as above from one group score per position:
 *
 *   s_g[t] = max_h s_h[t]                          (reduce = TB_GROUP_MAX)
 *   s_g[t] = ((s_0[t] + s_1[t]) + s_2[t]) + s_3[t] in fp32 (TB_GROUP_SUM)
 *
 * where s_h is the fp32 score of head h defined above.  Arguments, layouts,
 * limits and the workspace (tb_score_select_workspace_bytes) are those of
 * tb_score_select; idx, count and sel_bits receive the group's set in each of
 * its 4 heads' rows, so tb_sparse_decode_attn reads it unchanged.  Any other
 * reduce value is TB_ERR_INVALID_ARG. */
#define TB_GROUP_MAX 0
#define TB_GROUP_SUM 1
tb_status tb_score_select_group(const tb_dims *dims, const float *qp, int64_t qp_batch_stride,
                                const tb_bf16 *Kp, const int32_t *ctx_len, int32_t sink, int32_t window,
                                int32_t budget, int32_t nbr, int32_t reduce, int32_t *idx, int32_t idx_cap,
                                int32_t *count, uint32_t *sel_bits, void *ws, size_t ws_bytes,
                                void *stream);

/* Budget-inclusive variant (no counterpart on the pages; an alternative to
 * counting the budget before neighbour fetch).  Per query head, the
 * importance buffer itself holds at most `budget` positions: with the
 * candidates of C in the order (s desc, t asc) defined above,
 *
 *   I = ( ∪_{t in P} [t - nbr, t + nbr] ) ∩ C
 *
 * for the longest prefix P of that order whose I has at most `budget`
 * members (every member of P is in I, so |P| <= budget).  Arguments and
 * layouts are those of tb_score_select, except idx_cap >= min(budget,
 * ctx_cap) suffices; budget <= 8192 (larger is TB_ERR_UNSUPPORTED). */
tb_status tb_score_select_inclusive(const tb_dims *dims, const float *qp, int64_t qp_batch_stride,
                                    const tb_bf16 *Kp, const int32_t *ctx_len, int32_t sink, int32_t window,
                                    int32_t budget, int32_t nbr, int32_t *idx, int32_t idx_cap, int32_t *count,
                                    uint32_t *sel_bits, void *ws, size_t ws_bytes, void *stream);

/* The fp32 importance scores behind the last tb_score_select,
 * tb_score_select_group or tb_score_select_inclusive call made on `ws` with
 * the same dims, ctx_len, sink and window (the scoring step of "Core
 * architecture: scoring"), for inspection and for checking a selection
 * against the scores it was taken from:
 *
 *   scores[b][h][t] = s[t] of sequence b, query head h   for t in C = [sink, T - window)
 *                   = NaN                                 for every other t < ctx_cap
 *
 *   scores  [batch][Hq][ctx_cap] float (device)
 * After tb_score_select_group only the first head row of each KV head (h %
 * 4 == 0) holds the group scores; the other three rows are unspecified.  The
 * scores are the exact fp32 values the selection ranked.  Another selection
 * call on `ws` overwrites them. */
tb_status tb_score_select_scores(const tb_dims *dims, const void *ws, size_t ws_bytes, const int32_t *ctx_len,
                                 int32_t sink, int32_t window, float *scores, void *stream);

/* ---- selection algorithm -------------------------------------------------- */
/* Which kernels carry out tb_score_select and tb_score_select_group (the
 * result is the same, bit for bit: same scores, same set, same index list;
 * no counterpart on the pages, a choice of route):
 *
 *   TB_SELECT_AUTO          (default) the cluster route where one wave of
 *                           clusters holds the call with slices of at least
 *                           512 positions (few long sequences), else the
 *                           multi-kernel route.
 *   TB_SELECT_MULTI_KERNEL  three kernels per call: scoring with a histogram,
 *                           marking and candidate collection, and a per-head
 *                           finish (any ctx_cap).
 *   TB_SELECT_CLUSTER       two kernels per call: scoring on every SM, then a
 *                           thread-block cluster per (sequence, KV head) that
 *                           holds all of its scores on chip and selects.  It
 *                           applies while ctx_cap fits 16 CTAs (up to 131,072
 *                           positions for tb_score_select, 524,288 for
 *                           tb_score_select_group); elsewhere the selection
 *                           calls return TB_ERR_UNSUPPORTED.
 *
 * tb_score_select_inclusive always takes the multi-kernel path.  The
 * algorithm belongs to the calling thread and is read when a selection call
 * launches.  Any other value is TB_ERR_INVALID_ARG. */
#define TB_SELECT_AUTO 0
#define TB_SELECT_MULTI_KERNEL 1
#define TB_SELECT_CLUSTER 2
tb_status tb_select_set_algorithm(int32_t algorithm);
int32_t   tb_select_algorithm(void);

/* ---- context-parallel selection and attention ----------------------------- */
/* One sequence's context split over R ranks (each holds the K, V and K' rows
 * of a block of positions): the scale-out the survey of this path proposes
 * for contexts past 256K tokens.  No counterpart on the pages, which run on
 * one device; the result is the single-device result:
 *   1. each rank runs tb_score_select (nbr = 0) on its block, with the block's
 *      part of C as its candidates, so its set is exactly its local top-B;
 *   2. tb_select_export_candidates turns that set into composites
 *      (key << 32) | (0xFFFFFFFF - global position), key being the score's
 *      order-preserving image, which rank first in the (score desc, position
 *      asc) order; the ranks exchange them (an all-gather);
 *   3. tb_select_merge_candidates takes the top-B of all ranks' composites
 *      (every member of the global top-B is in its block's local top-B),
 *      applies the neighbour fetch and the clip to C on global positions, and
 *      gives each rank the rows of its block that the attention keeps;
 *   4. tb_sparse_decode_attn_partial attends over exactly those rows and
 *      returns each head's unnormalised softmax state; the ranks exchange
 *      them and tb_attn_combine merges them into the output.
 * Only per-head selection is supported (not the group-shared variant). */

/* Step 2.  For each (sequence b, query head h) of a rank's selection (dims,
 * ws and the idx/count it wrote, with nbr = 0), write its first
 * min(count[b][h], budget) positions p as composites of their score key and
 * p + pos_offset (the block's first global position):
 *   cand  [batch][Hq][budget] uint64 (device, 8-byte aligned); unused slots 0 */
tb_status tb_select_export_candidates(const tb_dims *dims, const void *ws, size_t ws_bytes, const int32_t *idx,
                                      int32_t idx_cap, const int32_t *count, int32_t budget, int32_t pos_offset,
                                      uint64_t *cand, void *stream);

/* Step 3, on every rank.  dims are the global shapes (ctx_cap = the global
 * capacity, a multiple of 32 is not needed); cand holds all ranks' exports,
 * [n_ranks][batch][Hq][budget].  With T = ctx_len[b] (global), C = [sink,
 * T - window):
 *   Top = the `budget` composites of (b, h) that rank first among those whose
 *         position lies in C (all of them if there are fewer)
 *   I   = ( ∪_{t in Top} [t - nbr, t + nbr] ) ∩ C         (global positions)
 *   idx [batch][Hq][idx_cap], count [batch][Hq]: I sorted, as tb_score_select
 *   local_bits [batch][Hq][ceil(local_cap/32)] uint32: bit t - shard_begin set
 *         for t in (sink ∪ window ∪ I) ∩ [shard_begin, shard_begin + shard_len)
 *         ∩ [0, T) (the rows this rank's partial attention reads)
 * shard_begin must be a multiple of 32; ws >= 256 bytes holds the flag word
 * (TB_FLAG_IDX_OVERFLOW, TB_FLAG_CTX_RANGE). */
tb_status tb_select_merge_candidates(const tb_dims *dims, const uint64_t *cand, int32_t n_ranks, int32_t budget,
                                     const int32_t *ctx_len, int32_t sink, int32_t window, int32_t nbr,
                                     int32_t *idx, int32_t idx_cap, int32_t *count, int32_t shard_begin,
                                     int32_t shard_len, int32_t local_cap, uint32_t *local_bits, void *ws,
                                     size_t ws_bytes, void *stream);

/* Step 4a.  The attention of tb_sparse_decode_attn over exactly the rows
 * whose bit is set (no sink or window of its own), rows[b] being the number
 * of valid rows of sequence b in this rank's cache (1 <= rows[b] <= ctx_cap),
 * returning per (b, h) the unnormalised state in log2 units:
 *   part[b][h][0..d)  = sum_t 2^(l_t - M) v_t,  part[b][h][d] = M = max_t l_t,
 *   part[b][h][d + 1] = sum_t 2^(l_t - M),      l_t = scale * log2(e) * q.k_t
 * (M = -inf and zeros when no row is kept).  part: [batch][Hq][d + 2] float. */
tb_status tb_sparse_decode_attn_partial(const tb_dims *dims, const tb_bf16 *Q, const tb_bf16 *K, const tb_bf16 *V,
                                        const int32_t *rows, const uint32_t *bits, float scale, float *part,
                                        void *ws, size_t ws_bytes, void *stream);

/* Step 4b.  out[b][h] = sum_p 2^(M_p - M*) o_p / sum_p 2^(M_p - M*) L_p over
 * n_parts states parts[p][b][h] (tb_sparse_decode_attn_partial's layout),
 * M* = max_p M_p; 0 when every part is empty.  out: [batch][Hq][head_dim]. */
tb_status tb_attn_combine(const float *parts, int32_t n_parts, int32_t batch, int32_t n_q_heads, int32_t head_dim,
                          float *out, void *stream);

/* Build the sel_bits bitmap from index lists that came from elsewhere (e.g. a
 * host-side selection): bit t of row (b,h) is set iff t is among
 * idx[b][h][0 .. count[b][h]).  Entries outside [0, ctx_cap) are ignored. */
tb_status tb_select_bits_from_idx(const tb_dims *dims, const int32_t *idx, int32_t idx_cap,
                                  const int32_t *count, uint32_t *sel_bits, void *stream);

/* ---- KV cache append ------------------------------------------------------ */
/* The full KV cache stays resident and attention reads the kept rows
 * (summary, "Significance"), so at every decode step the token being decoded
 * is appended to every layer's cache.  This writes, in one launch, for every
 * layer l < n_layers, sequence b and KV head g, with pos = ctx_len[b] - 1:
 *
 *   K_l[b][g][pos][:] = src[l][0][b][g][:],   V_l[b][g][pos][:] = src[l][1][b][g][:]
 *
 *   src      [n_layers][2][batch][Hkv][head_dim] bf16 (device, 16-byte aligned)
 *   caches   [2 * n_layers] uint64 device array of cache base addresses: K of
 *            layer l at 2l, V at 2l + 1, each [batch][Hkv][ctx_cap][head_dim]
 *            bf16, 16-byte aligned
 *   ctx_len  [batch] int32 (device): T including the token being decoded
 *   ws       any libtb workspace of at least 256 bytes (its flag word)
 * Rows whose pos lies outside [0, ctx_cap) are skipped and TB_FLAG_CTX_RANGE
 * is raised; a null or misaligned cache address is skipped with
 * TB_FLAG_BAD_CACHE.  No counterpart on the pages: the decode loop's cache
 * write, gathered into one call. */
tb_status tb_kv_append(const tb_dims *dims, int32_t n_layers, const tb_bf16 *src, const uint64_t *caches,
                       const int32_t *ctx_len, void *ws, size_t ws_bytes, void *stream);

/* ---- failure detection self-test ----------------------------------------- */
/* Every wait inside the kernels is bounded by a clock budget; when one runs
 * out the kernel raises TB_FLAG_TIMEOUT in the workspace flag word, leaves its
 * loops and returns, so the context stays usable.  This call exercises that
 * path on purpose: one thread waits on an mbarrier that nothing ever arrives
 * on, gives up after budget_cycles (1 .. 4e9) SM clock cycles and raises
 * TB_FLAG_TIMEOUT in ws (>= 256 bytes).  tb_workspace_check then reports it.
 * No counterpart on the pages. */
tb_status tb_selftest_bounded_wait(void *ws, size_t ws_bytes, int64_t budget_cycles, void *stream);

/* ---- 5. sparse GQA decode attention --------------------------------------- */
/* The full KV cache stays resident and only the selected tokens are read
 * (summary, "Significance"); the kept rows are sink ∪ local window ∪
 * importance buffer (summary, "Inference strategy").  For each sequence b and
 * query head h, with T = ctx_len[b]:
 *
 *   A   = [0, min(sink,T)) ∪ [max(sink, T-window), T) ∪ { t in [sink, T-window) :
 *         bit t of sel_bits[b][h] }
 *   out[b][h] = sum_{t in A} softmax_t( scale * Q[b][h]·K[b][g][t] ) * V[b][g][t]
 *
 * fp32 logits, fp32 online softmax, fp32 accumulation; every (b, KV head, t)
 * row is read once for the whole GQA group of 4 query heads, and a row in no
 * head's A is never read (its contents, NaN included, cannot reach out).
 *   Q    [batch][Hq][d] bf16;  K, V [batch][Hkv][ctx_cap][d] bf16
 *   out  [batch][Hq][d] fp32
 * Split over the context across CTAs; the last CTA of each (b, KV head) merges
 * the partial softmax states (no inter-CTA waiting). */
tb_status tb_sparse_decode_attn(const tb_dims *dims, const tb_bf16 *Q, const tb_bf16 *K,
                                const tb_bf16 *V, const int32_t *ctx_len, int32_t sink,
                                int32_t window, const uint32_t *sel_bits, float scale,
                                float *out, void *ws, size_t ws_bytes, void *stream);

/* ---- balanced attention slices -------------------------------------------- */
/* The attention splits each (sequence, KV head) over several CTAs.  By
 * default the slices are equal shares of the length T; the kept rows are not
 * spread evenly over the positions, so some slices hold more rows than
 * others and the launch lasts as long as the fullest.  A plan cuts the slices
 * at equal shares of the kept rows instead.  No counterpart on the pages: a
 * scheduling aid.
 *
 * tb_attn_plan counts, for each (b, KV head g), the kept rows of every
 * 32-position word below T = ctx_len[b] (sink ∪ window ∪ the positions
 * selected for any of the group's 4 query heads in sel_bits, as defined
 * under tb_sparse_decode_attn) and writes the word index at which each slice
 * opens:
 *   plan  [batch][Hkv][TB_ATTN_PLAN_STRIDE] int32 (device, 4-byte aligned):
 *         plan[b][g][s] for s = 0 .. splits, where splits is the attention's
 *         CTA count per (b, g) for these dims; entries past it are not written
 * The selection of an interval stays valid for its steps, and so does its
 * plan (the window's few moving rows only shift the balance slightly): run
 * tb_attn_plan once after each selection.
 *
 * tb_sparse_decode_attn_planned is tb_sparse_decode_attn with the slices of
 * `plan` (from tb_attn_plan with the same dims).  The result is the same up to
 * the order of the fp32 additions that merge the slices.  Under
 * TB_ATTN_PREFETCH_KV the plan is read before the preceding kernel has
 * completed, like sel_bits. */
#define TB_ATTN_PLAN_STRIDE 65
tb_status tb_attn_plan(const tb_dims *dims, const uint32_t *sel_bits, const int32_t *ctx_len, int32_t sink,
                       int32_t window, int32_t *plan, void *ws, size_t ws_bytes, void *stream);
tb_status tb_sparse_decode_attn_planned(const tb_dims *dims, const tb_bf16 *Q, const tb_bf16 *K,
                                        const tb_bf16 *V, const int32_t *ctx_len, int32_t sink,
                                        int32_t window, const uint32_t *sel_bits, const int32_t *plan,
                                        float scale, float *out, void *ws, size_t ws_bytes, void *stream);

/* ---- attention launch mode ------------------------------------------------ */
/* How the attention entry points (tb_sparse_decode_attn, tb_decode_attn,
 * tb_sparse_decode_attn_noalloc) order their reads against the kernel that
 * precedes them in the stream.  Every libtb kernel is launched with
 * programmatic stream serialization, so its CTAs may start while that kernel
 * is still finishing.  No counterpart on the pages: a launch option.
 *
 *   TB_ATTN_WAIT_ALL     (default) nothing in global memory is touched before
 *                        the preceding kernel has completed.
 *   TB_ATTN_PREFETCH_KV  ctx_len, sel_bits (and the plan, for the planned
 *                        entry point) and the K and V rows below
 *                        ctx_len[b] - 1 are read (and the first tiles of K/V
 *                        streamed into shared memory) as soon as the kernel
 *                        is resident; Q, row ctx_len[b] - 1, out and the
 *                        workspace only after the preceding kernel has
 *                        completed.  Valid only when no kernel that may still
 *                        be running writes ctx_len, sel_bits, the plan or
 *                        those K/V rows: the kernel that immediately precedes the call
 *                        in its stream (a decode loop's Q/K/V projection
 *                        writes Q and row ctx_len[b] - 1 only, which is
 *                        allowed), and, if that kernel lets its own
 *                        dependents start before it has waited for its
 *                        predecessor, that predecessor too (libtb's kernels
 *                        never do).  The reads of the next tiles then overlap
 *                        the end of the preceding kernel.  A preceding kernel
 *                        that runs longer than about 2 s makes the bounded
 *                        waits give up (TB_FLAG_TIMEOUT).
 *
 * The mode belongs to the calling thread and is read when an attention call
 * launches (a graph captures it with the launch).  Any other value is
 * TB_ERR_INVALID_ARG. */
#define TB_ATTN_WAIT_ALL 0
#define TB_ATTN_PREFETCH_KV 1
tb_status tb_attn_set_launch_mode(int32_t mode);
int32_t   tb_attn_launch_mode(void);

/* ---- dense decode attention (comparator) ---------------------------------- */
/* The same computation over A = [0, T): the dense attention baseline the
 * summaries' on-GPU speedup is measured against ("Contributions 4").  Rows at
 * or past T are never read. */
tb_status tb_decode_attn(const tb_dims *dims, const tb_bf16 *Q, const tb_bf16 *K,
                         const tb_bf16 *V, const int32_t *ctx_len, float scale, float *out,
                         void *ws, size_t ws_bytes, void *stream);

/* ---- sparse decode attention without a workspace ------------------------- */
/* No counterpart in the paper: an integration convenience of this library.
 * For callers that cannot allocate device memory for the call — a plugin or
 * custom-operator boundary that is handed only its inputs and outputs, or a
 * decode loop that must not call cudaMalloc on the hot path because it can
 * synchronise the whole device.  Same arguments and result as
 * tb_sparse_decode_attn, minus the workspace: the scratch is one fixed,
 * file-scope device array of TB_NOALLOC_SCRATCH_BYTES that every GPU loading
 * the library keeps until the process exits.
 *  - Limit: dims whose tb_attn_workspace_bytes() exceeds
 *    TB_NOALLOC_SCRATCH_BYTES are rejected with TB_ERR_WORKSPACE (at
 *    head_dim 128 that is at most 31 (sequence, KV head) pairs).
 *  - The first call on a device sets the scratch up (address lookup and a
 *    synchronous clear); make that first call before any stream capture.
 *  - All calls on a device share the scratch: calls that overlap on the GPU
 *    race and give wrong outputs.  Device-side flags are not reported.
 *  - Nothing is allocated or freed. */
#define TB_NOALLOC_SCRATCH_BYTES (4u << 20)
tb_status tb_sparse_decode_attn_noalloc(const tb_dims *dims, const tb_bf16 *Q, const tb_bf16 *K,
                                        const tb_bf16 *V, const int32_t *ctx_len, int32_t sink,
                                        int32_t window, const uint32_t *sel_bits, float scale,
                                        float *out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* TB_H */
