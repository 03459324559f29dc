/*
 * TokenButler decode-path oracle: plain, slow, single-threaded C in double
 * precision.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link,
 * load or call this file.  It is used by the tests, by the package smoke check
 * and by the CPU-baseline leg of the benchmark, and by nothing else.  It shares
 * no code, header, table or helper with the CUDA library.
 *
 * Sources (cited by page title and section):
 *   [ja]  "技術概要：TokenButler" (gist.science, Japanese summary of
 *         arXiv 2503.07518), sections コアアーキテクチャ (core architecture),
 *         推論戦略 (inference strategy) and 最適化 (optimisations).
 *   [ko]  "기술 요약: TokenButler" (gist.science, Korean summary of the same
 *         paper), sections 핵심 아키텍처 and 추론 전략 — same content, used as
 *         corroboration.
 *
 * The pages give prose only.  Every place where they leave a step open is
 * resolved by a stated reading (R1..R11 below); the same readings are listed in
 * the design notes of the repository.
 *
 *   R1  selection is per query head; projected keys are per KV head.
 *   R3  the budget B counts the top-scored tokens before neighbour fetch.
 *   R4  sink = [0, min(S,T)), window = [max(S,T-N), T), candidates C = [S, T-N).
 *   R6  K, V, Q, weights, h are bf16; K' is stored bf16 (round to nearest even);
 *       q', scores, softmax and outputs are fp32; the MLP hidden activation is
 *       rounded to bf16 between the two matrix products; no biases.
 *   R7  softmax scale is given by the caller (1/sqrt(d) in every workload).
 *   R9  ties in the top-B order go to the lower position.
 *
 * Precision policy.  Every sum is taken in double.  Where a floating-point
 * value decides an integer result -- the bf16 code of a projected key or of the
 * MLP activation, and the order of scores in the top-B -- the oracle takes the
 * decision in the precision the data path stores: K' and the activation are
 * rounded from the double sum to bf16, and scores are rounded from the double
 * sum to fp32 before they are compared.
 *
 * Parity pins: see the oracle pin tests.  Every function below is pinned
 * except where its comment says "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* bf16 <-> double                                                           */
/* ------------------------------------------------------------------------ */

/* A bf16 value is the upper 16 bits of an IEEE-754 binary32 value; widening
 * is exact. */
double orc_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 value, ties to even, in one step (no
 * intermediate rounding to binary32, which could round twice).  bf16 keeps 8
 * significant bits and the binary32 exponent range, with subnormals down to
 * 2^-133.  Values past the largest finite bf16 after rounding become inf. */
uint16_t orc_double_to_bf16(double x)
{
    if (isnan(x)) return (uint16_t)0x7fc0;
    double ax = fabs(x);
    uint16_t sign = signbit(x) ? (uint16_t)0x8000 : (uint16_t)0;
    if (ax == 0.0) return sign;
    if (isinf(x)) return (uint16_t)(sign | 0x7f80);

    int e;
    (void)frexp(ax, &e);                 /* ax = m * 2^e, m in [0.5, 1) */
    /* quantum = 2^(e-8) for normals (8 significant bits); clamp at the
     * subnormal quantum 2^-133 */
    int qexp = e - 8;
    if (qexp < -133) qexp = -133;
    double scaled = ldexp(ax, -qexp);    /* exact: power-of-two scaling */
    double r = nearbyint(scaled);        /* default mode: nearest, ties even */
    double v = ldexp(r, qexp);
    if (v > 3.38953138925153547590470800371487866880e+38) /* max finite bf16 */
        return (uint16_t)(sign | 0x7f80);
    float f = (float)v;                  /* exact: v is a bf16 value */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | ((u >> 16) & 0x7fff));
}

/* ------------------------------------------------------------------------ */
/* Step 1: key-cache projection                                              */
/* [ja] コアアーキテクチャ, キーキャッシュ射影: each consumer layer projects its  */
/* real keys with a learned matrix into the low-dimensional space; [ja] 最適化, */
/* バッチ処理: the projection runs on batches of N tokens.  The batching is a     */
/* schedule property (which rows are projected when); the per-row arithmetic  */
/* is the plain product below.                                               */
/* ------------------------------------------------------------------------ */

/* Kp[t][j] = bf16( sum_i K[t][i] * Wk[j][i] ),  t in [0, rows), j in [0, dp).
 * K is [rows][d], Wk is [dp][d] (output-major, one matrix per KV head),
 * Kp is [rows][dp]. */
void orc_project_keys(const uint16_t *K, const uint16_t *Wk, uint16_t *Kp,
                      int64_t rows, int d, int dp)
{
    for (int64_t t = 0; t < rows; ++t) {
        for (int j = 0; j < dp; ++j) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i)
                acc += orc_bf16_to_double(K[t * d + i]) *
                       orc_bf16_to_double(Wk[(int64_t)j * d + i]);
            Kp[t * dp + j] = orc_double_to_bf16(acc);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Step 2: query prediction                                                  */
/* [ja] コアアーキテクチャ, クエリ予測: a light MLP takes the producer layer's   */
/* hidden state and emits G slot-specific low-dimensional queries per head.   */
/* Reading R6: two bias-free matrix products with SiLU between them, the      */
/* activation rounded to bf16 before the second product.                      */
/* ------------------------------------------------------------------------ */

/* h: [batch][hidden]; W1: [inter][hidden]; W2: [n_out][inter];
 * qp: [batch][n_out] with n_out = G * Hq * d'. */
void orc_predict_queries(const uint16_t *h, const uint16_t *W1, const uint16_t *W2,
                         float *qp, int batch, int hidden, int inter, int n_out)
{
    uint16_t *act = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)inter);
    for (int b = 0; b < batch; ++b) {
        for (int i = 0; i < inter; ++i) {
            double a = 0.0;
            for (int k = 0; k < hidden; ++k)
                a += orc_bf16_to_double(h[(int64_t)b * hidden + k]) *
                     orc_bf16_to_double(W1[(int64_t)i * hidden + k]);
            double silu = a / (1.0 + exp(-a));  /* SiLU(a) = a * sigmoid(a) */
            act[i] = orc_double_to_bf16(silu);
        }
        for (int o = 0; o < n_out; ++o) {
            double q = 0.0;
            for (int i = 0; i < inter; ++i)
                q += orc_bf16_to_double(act[i]) *
                     orc_bf16_to_double(W2[(int64_t)o * inter + i]);
            qp[(int64_t)b * n_out + o] = (float)q;
        }
    }
    free(act);
}

/* ------------------------------------------------------------------------ */
/* Step 3: importance scores                                                 */
/* [ja] コアアーキテクチャ, スコアリング: the dot product of the predicted      */
/* query with each projected key is the token's importance score.             */
/* ------------------------------------------------------------------------ */

/* s[t - t_begin] = fp32( sum_j qp[j] * Kp[t][j] ) for t in [t_begin, t_end).
 * Kp is the [rows][dp] projected-key array of one KV head. */
void orc_scores(const float *qp, const uint16_t *Kp, int dp,
                int64_t t_begin, int64_t t_end, float *s)
{
    for (int64_t t = t_begin; t < t_end; ++t) {
        double acc = 0.0;
        for (int j = 0; j < dp; ++j)
            acc += (double)qp[j] * orc_bf16_to_double(Kp[t * dp + j]);
        s[t - t_begin] = (float)acc;
    }
}

/* ------------------------------------------------------------------------ */
/* Step 3, group-shared variant (not on the pages).                          */
/* An alternative to reading R1 in which the G query heads of a GQA group    */
/* share one importance set, chosen from one group score per position: the   */
/* largest (reduce = 0) or the sum (reduce = 1) of the heads' fp32 scores.    */
/* Each head's score is exactly the fp32 score of orc_scores; the sum is     */
/* taken in fp32 in head order, ((s0 + s1) + s2) + ..., which is the value a */
/* device that holds fp32 head scores and adds them in that order computes.  */
/* qp holds the G heads' projected queries, [G][dp].                          */
/* ------------------------------------------------------------------------ */

void orc_group_scores(const float *qp, int G, const uint16_t *Kp, int dp,
                      int64_t t_begin, int64_t t_end, int reduce, float *s)
{
    for (int64_t t = t_begin; t < t_end; ++t) {
        float g = 0.0f;
        for (int h = 0; h < G; ++h) {
            double acc = 0.0;
            for (int j = 0; j < dp; ++j)
                acc += (double)qp[(int64_t)h * dp + j] * orc_bf16_to_double(Kp[t * dp + j]);
            const float sh = (float)acc;
            if (h == 0)
                g = sh;
            else if (reduce == 0)
                g = sh > g ? sh : g;
            else
                g = g + sh;
        }
        s[t - t_begin] = g;
    }
}

/* ------------------------------------------------------------------------ */
/* Step 4: budgeted selection with neighbour fetch                           */
/* [ja] コアアーキテクチャ, スコアリング: dynamic token selection under a fixed */
/* budget.  [ja] 推論戦略: the first S tokens (sink) and the last N tokens     */
/* (local window) are always kept; the importance buffer is filled from the    */
/* predicted scores.  [ja] 最適化, 予測間隔と近隣取得: the selected tokens are  */
/* expanded by their spatial neighbours.                                       */
/*                                                                            */
/* Readings: candidates C = [S, T-N) (R4); Top = the B candidates that come   */
/* first in the order (score descending, position ascending) (R3, R9); the    */
/* importance set I = (union over t in Top of [t-r, t+r]) intersected with C; */
/* I is returned sorted ascending.                                            */
/* ------------------------------------------------------------------------ */

typedef struct { float s; int32_t t; } orc_cand;

static int orc_cand_cmp(const void *a, const void *b)
{
    const orc_cand *x = (const orc_cand *)a, *y = (const orc_cand *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->t < y->t) ? -1 : (x->t > y->t) ? 1 : 0;
}

/* s: scores of the candidates, s[k] belongs to position S + k, k < |C|.
 * Writes I into idx (capacity >= min(3B, |C|) for r = 1) and returns |I|. */
int64_t orc_select(const float *s, int64_t T, int64_t S, int64_t N, int64_t B,
                   int r, int32_t *idx)
{
    int64_t c_lo = S, c_hi = T - N;
    if (c_hi <= c_lo || B <= 0) return 0;
    int64_t nC = c_hi - c_lo;

    orc_cand *c = (orc_cand *)malloc(sizeof(orc_cand) * (size_t)nC);
    for (int64_t k = 0; k < nC; ++k) { c[k].s = s[k]; c[k].t = (int32_t)(c_lo + k); }
    qsort(c, (size_t)nC, sizeof(orc_cand), orc_cand_cmp);
    int64_t take = B < nC ? B : nC;

    unsigned char *keep = (unsigned char *)calloc((size_t)nC, 1);
    for (int64_t k = 0; k < take; ++k) {
        int64_t t = c[k].t;
        for (int64_t u = t - r; u <= t + r; ++u)
            if (u >= c_lo && u < c_hi) keep[u - c_lo] = 1;
    }
    int64_t n = 0;
    for (int64_t k = 0; k < nC; ++k)
        if (keep[k]) idx[n++] = (int32_t)(c_lo + k);
    free(keep);
    free(c);
    return n;
}

/* ------------------------------------------------------------------------ */
/* Step 4, budget-inclusive variant (not on the pages).  An alternative to    */
/* reading R3 in which the importance buffer itself holds at most B tokens:  */
/* candidates are taken in the order of orc_select (score descending,        */
/* position ascending) while the union of their [t-r, t+r] neighbourhoods,   */
/* clipped to C, stays within B; the first candidate that would push it past */
/* B ends the selection.  Every taken candidate belongs to the union, so at  */
/* most B candidates are taken.                                               */
/* ------------------------------------------------------------------------ */

int64_t orc_select_inclusive(const float *s, int64_t T, int64_t S, int64_t N, int64_t B,
                             int r, int32_t *idx)
{
    const int64_t lo = S, hi = T - N;
    if (hi <= lo || B <= 0) return 0;
    const int64_t n_cand = hi - lo;

    orc_cand *order = (orc_cand *)malloc(sizeof(orc_cand) * (size_t)n_cand);
    for (int64_t k = 0; k < n_cand; ++k) { order[k].s = s[k]; order[k].t = (int32_t)(lo + k); }
    qsort(order, (size_t)n_cand, sizeof(orc_cand), orc_cand_cmp);

    unsigned char *in_set = (unsigned char *)calloc((size_t)n_cand, 1);
    int64_t size = 0;
    for (int64_t k = 0; k < n_cand; ++k) {
        const int64_t t = order[k].t;
        const int64_t from = t - r < lo ? lo : t - r;
        const int64_t to = t + r > hi - 1 ? hi - 1 : t + r;
        int64_t fresh = 0;
        for (int64_t u = from; u <= to; ++u) fresh += !in_set[u - lo];
        if (size + fresh > B) break;
        for (int64_t u = from; u <= to; ++u) in_set[u - lo] = 1;
        size += fresh;
    }
    int64_t n = 0;
    for (int64_t k = 0; k < n_cand; ++k)
        if (in_set[k]) idx[n++] = (int32_t)(lo + k);
    free(in_set);
    free(order);
    return n;
}

/* The attended set A = sink U window U I, sorted ascending ([ja] 推論戦略).
 * I must lie in C = [S, T-N), so the three parts are disjoint.  Returns |A|. */
int64_t orc_attention_set(int64_t T, int64_t S, int64_t N,
                          const int32_t *I, int64_t nI, int32_t *A)
{
    int64_t n = 0;
    int64_t sink_end = S < T ? S : T;
    int64_t win_begin = T - N > S ? T - N : S;
    for (int64_t t = 0; t < sink_end; ++t) A[n++] = (int32_t)t;
    for (int64_t k = 0; k < nI; ++k)
        if (I[k] >= sink_end && I[k] < win_begin) A[n++] = I[k];
    for (int64_t t = win_begin; t < T; ++t) A[n++] = (int32_t)t;
    return n;
}

/* ------------------------------------------------------------------------ */
/* Step 5: attention over the kept rows                                      */
/* [ja] 意義: the full KV cache stays resident and only the selected tokens    */
/* are read.  Standard scaled dot-product attention restricted to the rows in */
/* A (R7: no RoPE, no mask beyond A).  Two passes in double: max, then the    */
/* normalised weighted sum.                                                   */
/* ------------------------------------------------------------------------ */

/* q: [d]; K, V: [rows][d] of one KV head; A: n_rows row positions;
 * out: [d] fp32.  An empty A gives a zero output. */
void orc_attention(const uint16_t *q, const uint16_t *K, const uint16_t *V, int d,
                   const int32_t *A, int64_t n_rows, double scale, float *out)
{
    if (n_rows <= 0) { for (int j = 0; j < d; ++j) out[j] = 0.0f; return; }
    double *z = (double *)malloc(sizeof(double) * (size_t)n_rows);
    double zmax = -INFINITY;
    for (int64_t k = 0; k < n_rows; ++k) {
        int64_t t = A[k];
        double acc = 0.0;
        for (int j = 0; j < d; ++j)
            acc += orc_bf16_to_double(q[j]) * orc_bf16_to_double(K[t * d + j]);
        z[k] = acc * scale;
        if (z[k] > zmax) zmax = z[k];
    }
    double l = 0.0;
    for (int64_t k = 0; k < n_rows; ++k) { z[k] = exp(z[k] - zmax); l += z[k]; }
    for (int j = 0; j < d; ++j) {
        double o = 0.0;
        for (int64_t k = 0; k < n_rows; ++k)
            o += z[k] * orc_bf16_to_double(V[(int64_t)A[k] * d + j]);
        out[j] = (float)(o / l);
    }
    free(z);
}
