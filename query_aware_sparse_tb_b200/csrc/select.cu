// Importance scoring and budgeted top-B selection with neighbour fetch.
//
// TokenButler technical summary (gist.science), "Core architecture: scoring":
// the predicted queries are dot-multiplied with the projected keys to give
// cheap per-token importance scores, which drive a dynamic token selection
// under a fixed budget.  "Inference strategy": the first S tokens (sink) and
// the last N tokens (local window) are always kept, so the candidates are
// C = [S, T-N).  "Optimisations: prediction interval and neighbour fetch": the
// selected tokens are expanded by their spatial neighbours.
//
// Exact top-B on the fp32 scores, ties broken by the lower position:
//   1. score_hist   one CTA per (b, KV head, 2048 positions; without the
//                   histogram, chunks sized for two CTAs per SM): each warp
//                   streams 32-row blocks of K' through a cp.async ring of its
//                   own and scores each row once for the 4 query heads of the
//                   group (BlockScorer), writes the
//                   order-preserving uint32 image of every score, and builds
//                   a histogram of its top 11 bits per query head.  The last
//                   CTA of each (b, KV head) (atomic ticket, no waiting) finds
//                   the bin that holds the B-th largest key.
//   2. mark_collect same grid: keys above that bin become bits of the Top
//                   bitmap; keys inside it go to a per-head candidate list.
//   3. finalize     one CTA per (b, query head): two more 11/10-bit radix
//                   passes over the candidate list fix the B-th key exactly,
//                   ties on it are taken in position order, and the Top bitmap
//                   is dilated by +-nbr, clipped to C, and written out both as
//                   the bitmap and as the sorted index list.
//
// Two variants share the kernels through a template mode (no counterpart on
// the pages): one set per KV head from the max or the fp32 sum of the
// group's head scores (the kernels then work on one row per group and
// finalize copies the set to the group's 4 heads), and a budget that includes
// the neighbours (finalize keeps the longest prefix of the top-B, in score
// order, whose neighbourhoods cover at most B positions, found with a radix
// select over the candidates' composites weighted by what each one adds).
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "score.cuh"
#include "select_common.cuh"

namespace tb {
namespace {

using namespace sel;

// ------------------------------------------------------------------ kernel 1

// HIST = false: the scores only (their keys in the workspace), for the
// cluster kernel that selects from them.
template <int DP, int SEL, bool HIST>
__global__ void __launch_bounds__(kThreads, 2)
score_hist_kernel(const float *__restrict__ qp, int64_t qp_stride, const uint16_t *__restrict__ Kp,
                  const int32_t *__restrict__ ctx_len, int Hq, int Hkv, int Tcap, int sink,
                  int window, int budget, int chunk, SelWs ws) {
    constexpr int NH = sel_is_group(SEL) ? 1 : kGroup;  // score rows per (b, KV head)
    using Sc = BlockScorer<DP>;
    constexpr int NW = kThreads / 32;
    constexpr int RING = hist_ring(HIST);
    extern __shared__ __align__(128) uint8_t stage[];   // [warp][RING][32-row block]
    __shared__ __align__(16) float qs[kGroup][DP];
    __shared__ uint32_t hist[HIST ? NH : 1][HIST ? kBins1 : 1];
    __shared__ int s_last;
    __shared__ int scratch[kThreads / 32 + 3];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.z, g = blockIdx.y, ch = blockIdx.x;
    const int p0 = ch * chunk;  // this CTA's positions: [p0, p0 + chunk), chunk a multiple of 32

    if constexpr (HIST)
        for (int i = tid; i < NH * kBins1; i += kThreads) (&hist[0][0])[i] = 0u;
    griddep_wait();
    griddep_launch_dependents();
    const int T = clamp_ctx(ctx_len[b], Tcap, ws.flags, tid == 0 && ch == 0 && g == 0);
    const int lo = sink, hi = T - window;
    if (tid < kGroup * DP) (&qs[0][0])[tid] = qp[(int64_t)b * qp_stride + (int64_t)g * kGroup * DP + tid];
    __syncthreads();

    const size_t slab = ((size_t)b * Hkv + g) * (size_t)Tcap;
    if (hi > lo && p0 < hi && p0 + chunk > lo) {
        // the chunk's 32-row blocks that overlap C, dealt to the warps in
        // turn; each warp streams its blocks through a ring of its own
        // (RING - 1 in flight) and lane l scores row l of each
        const int blo = max(0, lo - p0) / 32;
        const int bhi = min(chunk, hi - p0 + 31) / 32;
        const int nb = blo + warp < bhi ? (bhi - blo - warp + NW - 1) / NW : 0;  // this warp's blocks
        uint8_t *ring = stage + warp * RING * Sc::BLKB;
        const uint32_t ring_s = smem_addr(ring);
        auto issue = [&](int i) {
            const int r0 = p0 + (blo + warp + NW * i) * 32;
            Sc::copy(ring_s + (uint32_t)((i % RING) * Sc::BLKB), Kp + (slab + r0) * DP, hi - r0, lane);
        };
        // blocks go in pairs: RING - 2 in flight beside the pair being scored
        static_assert(RING % 2 == 0, "pairs of slots");
        for (int i = 0; i < RING - 2; ++i) {
            if (i < nb) issue(i);
            cp_async_commit();
        }
        auto emit = [&](int i, const float *sc) {  // block i's keys (and histogram)
            const int p = p0 + (blo + warp + NW * i) * 32 + lane;
            const bool valid = p >= lo && p < hi;
            if constexpr (!sel_is_group(SEL)) {
#pragma unroll
                for (int h = 0; h < kGroup; ++h) {
                    const uint32_t key = score_key(sc[h]);
                    if (valid) {
                        ws.keys[((size_t)b * Hq + g * kGroup + h) * Tcap + p] = key;
                        if constexpr (HIST) atomicAdd(&hist[h][key >> 21], 1u);
                    }
                }
            } else {
                float gs = sc[0];
#pragma unroll
                for (int h = 1; h < kGroup; ++h) gs = SEL == kSelGroupMax ? fmaxf(gs, sc[h]) : gs + sc[h];
                const uint32_t key = score_key(gs);
                if (valid) {
                    ws.keys[((size_t)b * Hq + g * kGroup) * Tcap + p] = key;
                    if constexpr (HIST) atomicAdd(&hist[0][key >> 21], 1u);
                }
            }
        };
        for (int i = 0; i < nb; i += 2) {
            if (i + RING - 2 < nb) issue(i + RING - 2);
            cp_async_commit();
            if (i + RING - 1 < nb) issue(i + RING - 1);
            cp_async_commit();
            cp_async_wait_group<RING - 2>();
            __syncwarp();  // every lane's copies of blocks i and i + 1 have landed
            float sa[kGroup], sb[kGroup];
            if (i + 1 < nb) {
                Sc::score2(ring + (i % RING) * Sc::BLKB, ring + ((i + 1) % RING) * Sc::BLKB, &qs[0][0], lane, sa, sb);
            } else {
                Sc::score(ring + (i % RING) * Sc::BLKB, &qs[0][0], lane, sa);
            }
            __syncwarp();  // the blocks are read before their slots are refilled
            emit(i, sa);
            if (i + 1 < nb) emit(i + 1, sb);
        }
    }
    if constexpr (!HIST) return;
    __syncthreads();
    for (int i = tid; i < NH * kBins1; i += kThreads) {
        const uint32_t v = (&hist[0][0])[i];
        if (v) atomicAdd(ws.hist + ((size_t)b * Hq + g * kGroup + i / kBins1) * kBins1 + (i % kBins1), v);
    }

    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(ws.counters + b * Hkv + g, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    const int nC = hi > lo ? hi - lo : 0;
    const uint32_t *gh0 = ws.hist + ((size_t)b * Hq + g * kGroup) * kBins1;
    if (nC > budget) {
        // thread t owns bins [hi_t - PERB, hi_t) of each head's histogram,
        // counted from the top; all loads first, then one scan per head
        constexpr int PERB = kBins1 / kThreads;
        const int hb = kBins1 - tid * PERB;
        uint32_t v[NH][PERB];
#pragma unroll
        for (int h = 0; h < NH; ++h)
#pragma unroll
            for (int j = 0; j < PERB; ++j) v[h][j] = __ldcg(gh0 + (size_t)h * kBins1 + hb - 1 - j);
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            int mine = 0;
#pragma unroll
            for (int j = 0; j < PERB; ++j) mine += (int)v[h][j];
            int total;
            const int above = block_excl_scan<kThreads>(mine, scratch, &total);
            if ((uint32_t)above < (uint32_t)budget && (uint32_t)budget <= (uint32_t)(above + mine)) {
                uint32_t acc = (uint32_t)above;
#pragma unroll
                for (int j = 0; j < PERB; ++j) {
                    if (acc + v[h][j] >= (uint32_t)budget) {
                        HeadState st = {};
                        st.mode = kModeSelect;
                        st.b1 = (uint32_t)(hb - 1 - j);
                        st.k_rem = (uint32_t)budget - acc;
                        st.n_in_bin = v[h][j];
                        ws.state[(size_t)b * Hq + g * kGroup + h] = st;
                        break;
                    }
                    acc += v[h][j];
                }
            }
        }
    } else if (tid < NH) {
        HeadState st = {};
        st.mode = nC == 0 ? kModeEmpty : kModeAll;
        ws.state[(size_t)b * Hq + g * kGroup + tid] = st;
    }
    __syncthreads();
    for (int i = tid; i < NH * kBins1; i += kThreads) ws.hist[((size_t)b * Hq + g * kGroup) * kBins1 + i] = 0u;
    if (tid == 0) ws.counters[b * Hkv + g] = 0u;
}

// ------------------------------------------------------------------ kernel 2

template <int SEL>
__global__ void __launch_bounds__(kThreads)
mark_collect_kernel(const int32_t *__restrict__ ctx_len, int Hq, int Hkv, int Tcap, int W,
                    int sink, int window, SelWs ws) {
    constexpr int kWordsPerWarp = kChunk / 32 / (kThreads / 32);  // 4
    constexpr int NH = sel_is_group(SEL) ? 1 : kGroup;
    __shared__ uint32_t s_cnt[kGroup], s_base[kGroup];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.z, g = blockIdx.y, ch = blockIdx.x;
    if (tid < kGroup) s_cnt[tid] = 0u;
    griddep_wait();
    griddep_launch_dependents();
    const int T = clamp_ctx(ctx_len[b], Tcap, ws.flags, false);
    const int lo = sink, hi = T - window;
    const int w0 = ch * (kChunk / 32);

    uint32_t mode[NH], b1[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) {
        const HeadState &st = ws.state[(size_t)b * Hq + g * kGroup + h];
        mode[h] = st.mode;
        b1[h] = st.b1;
    }
    __syncthreads();
    // pass 1: Top bits, candidate ballots and this warp's offsets inside the CTA
    // (every key load issued before the first ballot)
    uint32_t key[kWordsPerWarp][NH], cb[kWordsPerWarp][NH], off[kWordsPerWarp][NH];
#pragma unroll
    for (int i = 0; i < kWordsPerWarp; ++i) {
        const int w = w0 + warp + i * (kThreads / 32);
        const int p = (w << 5) + lane;
        const bool in_c = w < W && p >= lo && p < hi;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            const size_t row = (size_t)b * Hq + g * kGroup + h;
            key[i][h] = (in_c && mode[h] == kModeSelect) ? __ldcg(ws.keys + row * Tcap + p) : 0u;
        }
    }
#pragma unroll
    for (int i = 0; i < kWordsPerWarp; ++i) {
        const int w = w0 + warp + i * (kThreads / 32);
        const int p = (w << 5) + lane;
        const bool in_c = w < W && p >= lo && p < hi;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            const size_t row = (size_t)b * Hq + g * kGroup + h;
            const uint32_t k = key[i][h];
            const uint32_t d1 = k >> 21;
            const bool top = in_c && (mode[h] == kModeAll || (mode[h] == kModeSelect && d1 > b1[h]));
            const bool cand = in_c && mode[h] == kModeSelect && d1 == b1[h];
            const uint32_t tb = __ballot_sync(kFull, top);
            if (lane == 0 && w < W) ws.top[row * W + w] = tb;
            cb[i][h] = __ballot_sync(kFull, cand);
            uint32_t o = 0;
            if (lane == 0 && cb[i][h]) o = atomicAdd(&s_cnt[h], (uint32_t)__popc(cb[i][h]));
            off[i][h] = __shfl_sync(kFull, o, 0);
        }
    }
    __syncthreads();
    if (tid < NH && s_cnt[tid])
        s_base[tid] = atomicAdd(&ws.state[(size_t)b * Hq + g * kGroup + tid].cand_count, s_cnt[tid]);
    __syncthreads();
    // pass 2: the candidates, (key, position) pairs, in the reserved range
#pragma unroll
    for (int i = 0; i < kWordsPerWarp; ++i) {
        const int p = ((w0 + warp + i * (kThreads / 32)) << 5) + lane;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            if ((cb[i][h] >> lane) & 1u) {
                const size_t row = (size_t)b * Hq + g * kGroup + h;
                ws.cand[row * Tcap + s_base[h] + off[i][h] + __popc(cb[i][h] & ((1u << lane) - 1u))] =
                    ((unsigned long long)key[i][h] << 32) | (uint32_t)p;
            }
        }
    }
}

// ------------------------------------------------------------------ kernel 3


// One CTA per (b, query head) (per KV head in the group modes) of NT threads:
// 1024 on the default path, 512 for the variants, which need more registers.
template <int SEL>
__host__ __device__ constexpr int fin_threads() { return SEL == kSelHead ? kFinThreads : kFinThreads / 2; }

template <int SEL>
__global__ void __launch_bounds__(fin_threads<SEL>())
finalize_kernel(const int32_t *__restrict__ ctx_len, int Hq, int Tcap, int W, int sink, int window,
                int budget, int nbr, int32_t *__restrict__ idx, int idx_cap, int32_t *__restrict__ count,
                uint32_t *__restrict__ sel_bits, SelWs ws) {
    constexpr int NT = fin_threads<SEL>();
    extern __shared__ unsigned long long fsm8[];
    unsigned long long *cand_s = fsm8;                                  // [kCandCache]
    uint32_t *top_s = reinterpret_cast<uint32_t *>(fsm8 + kCandCache);  // [W]
    uint32_t *tie_s = top_s + W;                                        // [W]
    __shared__ uint32_t hist[kBins2];
    __shared__ int scratch[NT / 32 + 3];

    // a group's set is computed in its first head's rows and written to all 4
    constexpr int NOUT = sel_is_group(SEL) ? kGroup : 1;
    const int tid = threadIdx.x;
    const int h = blockIdx.x * NOUT, b = blockIdx.y;
    griddep_wait();
    griddep_launch_dependents();
    const size_t row = (size_t)b * Hq + h;
    const int T = clamp_ctx(ctx_len[b], Tcap, ws.flags, false);
    const int lo = sink, hi = T - window;
    const HeadState st = ws.state[row];

    for (int w = tid; w < W; w += NT) {
        top_s[w] = ws.top[row * W + w];
        tie_s[w] = 0u;
    }
    if (st.mode == kModeSelect) {
        const int n = (int)st.cand_count;
        // the candidate list is read three times: stage it in shared memory
        // when it fits
        const unsigned long long *cand = ws.cand + row * Tcap;
        if (n <= kCandCache) {
            for (int i = tid; i < n; i += NT) cand_s[i] = cand[i];
            cand = cand_s;
        }
        // digit 2: key bits 20..10 inside bin b1
        for (int i = tid; i < kBins2; i += NT) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += NT) {
            const uint32_t key = (uint32_t)(cand[i] >> 32);
            atomicAdd(&hist[(key >> 10) & 0x7FFu], 1u);
        }
        __syncthreads();
        uint32_t k2;
        const uint32_t b2 = (uint32_t)block_find_bin_desc<NT>(hist, kBins2, st.k_rem, &k2, scratch, false);
        // digit 3: key bits 9..0 inside (b1, b2)
        for (int i = tid; i < kBins3; i += NT) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += NT) {
            const uint32_t key = (uint32_t)(cand[i] >> 32);
            if (((key >> 10) & 0x7FFu) == b2) atomicAdd(&hist[key & 0x3FFu], 1u);
        }
        __syncthreads();
        uint32_t k3;  // keys equal to tau still to take, lowest positions first
        const uint32_t b3 = (uint32_t)block_find_bin_desc<NT>(hist, kBins3, k2, &k3, scratch, false);
        const uint32_t tau = (st.b1 << 21) | (b2 << 10) | b3;
        for (int i = tid; i < n; i += NT) {
            const unsigned long long e = cand[i];
            const uint32_t key = (uint32_t)(e >> 32), p = (uint32_t)e;
            if (key > tau) atomicOr(&top_s[p >> 5], 1u << (p & 31));
            else if (key == tau) atomicOr(&tie_s[p >> 5], 1u << (p & 31));
        }
        __syncthreads();
        // ties in position order: each thread owns a contiguous run of words
        const int wpt = (W + NT - 1) / NT;
        const int wb = tid * wpt, we = min(wb + wpt, W);
        int mine = 0;
        for (int w = wb; w < we; ++w) mine += __popc(tie_s[w]);
        int tot;
        int before = block_excl_scan<NT>(mine, scratch, &tot);
        for (int w = wb; w < we; ++w) {
            uint32_t t = tie_s[w];
            const int pc = __popc(t);
            uint32_t keep = 0u;
            if (before + pc <= (int)k3) {
                keep = t;
            } else if (before < (int)k3) {
                for (int k = 0; k < (int)k3 - before; ++k) {
                    const uint32_t low = t & (0u - t);
                    keep |= low;
                    t ^= low;
                }
            }
            top_s[w] |= keep;
            before += pc;
        }
    }
    __syncthreads();

    if constexpr (SEL == kSelInclusive) {
        // top_s holds the exact top-B positions (B <= kCandCache).  Keep the
        // longest prefix of them in score order whose neighbourhoods, clipped
        // to C, cover at most B positions.
        const int lane = tid & 31;
        const uint32_t lt = (1u << lane) - 1u;
        const uint32_t *keys = ws.keys + row * Tcap;
        // gain of the k-th top position (position order): after the tie
        // buffer, which now holds the per-word count of top positions before it
        uint16_t *gain_s = reinterpret_cast<uint16_t *>(tie_s + W);
        uint32_t *wpref = tie_s;
        // 1. gather (key, position) of the top positions, words in order
        const int wpt = (W + NT - 1) / NT;
        const int wb = tid * wpt, we = min(wb + wpt, W);
        int mine = 0;
        for (int w = wb; w < we; ++w) mine += __popc(top_s[w]);
        int n_top;
        const int base = block_excl_scan<NT>(mine, scratch, &n_top);
        {
            int acc = base;
            for (int w = wb; w < we; ++w) {
                wpref[w] = (uint32_t)acc;
                acc += __popc(top_s[w]);
            }
        }
        {
            // lane = bit; the keys of 16 words are requested before any is used
            constexpr int kWB = 16;
            const int w_first = (tid - lane) * wpt, w_last = min(w_first + 32 * wpt, W);
            int run = __shfl_sync(kFull, base, 0);
            for (int w0 = w_first; w0 < w_last; w0 += kWB) {
                uint32_t ev[kWB], kv[kWB];
#pragma unroll
                for (int u = 0; u < kWB; ++u) {
                    const int w = w0 + u;
                    ev[u] = w < w_last ? top_s[w] : 0u;
                    kv[u] = ((ev[u] >> lane) & 1u) ? __ldcg(keys + (w << 5) + lane) : 0u;
                }
#pragma unroll
                for (int u = 0; u < kWB; ++u) {
                    if ((ev[u] >> lane) & 1u) {
                        const uint32_t p = (uint32_t)(((w0 + u) << 5) + lane);
                        cand_s[run + __popc(ev[u] & lt)] = ((unsigned long long)kv[u] << 32) | (0xFFFFFFFFu - p);
                    }
                    run += __popc(ev[u]);
                }
            }
        }
        __syncthreads();
        // 2. gains, in position order: a top position ranks ahead of p exactly
        //    when its (key, inverted position) composite is larger, so no sort
        //    is needed to tell which neighbours come first
        auto top_index = [&](uint32_t u) {
            return wpref[u >> 5] + __popc(top_s[u >> 5] & ((1u << (u & 31)) - 1u));
        };
        auto is_top = [&](int u) { return (top_s[u >> 5] >> (u & 31)) & 1u; };
        uint32_t my_gain = 0;
        for (int j = tid; j < n_top; j += NT) {
            const unsigned long long cp = cand_s[j];
            const int p = (int)(0xFFFFFFFFu - (uint32_t)cp);
            uint32_t gain = 0;
            for (int q = max(p - nbr, lo); q <= min(p + nbr, hi - 1); ++q) {
                bool covered = false;
                for (int u = max(q - nbr, lo); u <= min(q + nbr, hi - 1) && !covered; ++u)
                    covered = is_top(u) && cand_s[top_index((uint32_t)u)] > cp;
                gain += covered ? 0u : 1u;
            }
            gain_s[j] = (uint16_t)gain;
            my_gain += gain;
        }
        int total_gain;
        (void)block_excl_scan<NT>((int)my_gain, scratch, &total_gain);
        // 3. the first candidate in score order whose running gain exceeds B:
        //    MSB-first radix over its 64-bit composite, weighted by the gains
        //    (six passes of 11/11/11/11/10/10 bits); the kept candidates are
        //    those ranked before it
        unsigned long long cut = 0ull;  // keep composites > cut (all of them if none exceeds B)
        if (total_gain > budget) {
            uint32_t need = (uint32_t)budget + 1u;
            unsigned long long prefix = 0ull;
            int fixed = 0;
#pragma unroll 1
            for (int pass = 0; pass < 6; ++pass) {
                const int dw = pass < 4 ? 11 : 10;
                const int nb = 1 << dw;
                const int shift = 64 - fixed - dw;
                for (int i = tid; i < nb; i += NT) hist[i] = 0u;
                __syncthreads();
                for (int j = tid; j < n_top; j += NT) {
                    const unsigned long long cp = cand_s[j];
                    if (fixed == 0 || (cp >> (64 - fixed)) == prefix)
                        atomicAdd(&hist[(uint32_t)(cp >> shift) & (uint32_t)(nb - 1)], (uint32_t)gain_s[j]);
                }
                __syncthreads();
                uint32_t rem;
                const uint32_t bin = (uint32_t)block_find_bin_desc<NT>(hist, nb, need, &rem, scratch, false);
                prefix = (prefix << dw) | bin;
                fixed += dw;
                need = rem;
            }
            cut = prefix;
        }
        // the kept positions: composites above the cut (or all)
        for (int w = tid; w < W; w += NT) tie_s[w] = 0u;
        __syncthreads();
        for (int j = tid; j < n_top; j += NT) {
            const unsigned long long cp = cand_s[j];
            if (total_gain <= budget || cp > cut) {
                const uint32_t p = 0xFFFFFFFFu - (uint32_t)cp;
                atomicOr(&tie_s[p >> 5], 1u << (p & 31));
            }
        }
        __syncthreads();
        for (int w = tid; w < W; w += NT) top_s[w] = tie_s[w];
        __syncthreads();
    }

    // neighbour fetch, clip to C, emit bitmap and sorted index list
    const int wpt = (W + NT - 1) / NT;
    const int wb = tid * wpt, we = min(wb + wpt, W);
    int mine = 0;
    for (int w = wb; w < we; ++w) {
        const uint32_t t = top_s[w];
        const uint32_t pv = w > 0 ? top_s[w - 1] : 0u, nx = w + 1 < W ? top_s[w + 1] : 0u;
        uint32_t e = t;
        for (int k = 1; k <= nbr; ++k) e |= (t << k) | (pv >> (32 - k)) | (t >> k) | (nx << (32 - k));
        e &= range_mask(w, lo, hi);
        tie_s[w] = e;  // reuse as the output bitmap
        mine += __popc(e);
    }
    int total;
    const int base = block_excl_scan<NT>(mine, scratch, &total);
    for (int w = wb; w < we; ++w)
#pragma unroll
        for (int o = 0; o < NOUT; ++o) sel_bits[(row + o) * W + w] = tie_s[w];
    // the index list, lane-parallel: a warp walks its threads' words in
    // order (they are contiguous), lane = bit, one predicated store each
    {
        const int lane = tid & 31;
        const uint32_t lt = (1u << lane) - 1u;
        int32_t *out = idx + row * (size_t)idx_cap;
        const int w_first = (tid - lane) * wpt, w_last = min(w_first + 32 * wpt, W);
        int run = __shfl_sync(kFull, base, 0);
        for (int w = w_first; w < w_last; ++w) {
            const uint32_t e = tie_s[w];
            const int slot = run + __popc(e & lt);
            if (((e >> lane) & 1u) && slot < idx_cap) {
#pragma unroll
                for (int o = 0; o < NOUT; ++o) out[(size_t)o * idx_cap + slot] = (w << 5) + lane;
            }
            run += __popc(e);
        }
    }
    if (tid == 0) {
        if (total > idx_cap) raise_flag(ws.flags, TB_FLAG_IDX_OVERFLOW);
#pragma unroll
        for (int o = 0; o < NOUT; ++o) count[row + o] = total < idx_cap ? total : idx_cap;
    }
}

// ------------------------------------------------------ bitmap from indices

__global__ void __launch_bounds__(kFinThreads)
bits_from_idx_kernel(const int32_t *__restrict__ idx, int idx_cap, const int32_t *__restrict__ count,
                     int Hq, int Tcap, int W, uint32_t *__restrict__ sel_bits) {
    extern __shared__ uint32_t bsm[];
    const int tid = threadIdx.x;
    const size_t row = (size_t)blockIdx.y * Hq + blockIdx.x;
    for (int w = tid; w < W; w += kFinThreads) bsm[w] = 0u;
    griddep_wait();
    griddep_launch_dependents();
    __syncthreads();
    int n = count[row];
    n = n < 0 ? 0 : (n > idx_cap ? idx_cap : n);
    for (int i = tid; i < n; i += kFinThreads) {
        const int t = idx[row * idx_cap + i];
        if (t >= 0 && t < Tcap) atomicOr(&bsm[t >> 5], 1u << (t & 31));
    }
    __syncthreads();
    for (int w = tid; w < W; w += kFinThreads) sel_bits[row * W + w] = bsm[w];
}

// ------------------------------------------- context-parallel selection

// A rank's local top-B as exchangeable candidates: for each selected local
// position p (a selection with nbr = 0, so its set is exactly its top-B),
// the composite (key << 32) | (0xFFFFFFFF - (p + pos_offset)) of its score's
// order-preserving key and its global position.  Larger composites rank first
// (score desc, position asc); 0 pads the unused slots.
__global__ void __launch_bounds__(kThreads)
export_candidates_kernel(const uint32_t *__restrict__ keys, const int32_t *__restrict__ idx, int idx_cap,
                         const int32_t *__restrict__ count, int Hq, int Tcap, int budget, int pos_offset,
                         unsigned long long *__restrict__ cand) {
    const int h = blockIdx.x, b = blockIdx.y;
    const size_t row = (size_t)b * Hq + h;
    griddep_wait();
    griddep_launch_dependents();
    int n = count[row];
    n = n < 0 ? 0 : (n > idx_cap ? idx_cap : n);
    n = n < budget ? n : budget;
    for (int i = threadIdx.x; i < budget; i += kThreads) {
        unsigned long long c = 0ull;
        if (i < n) {
            const int p = idx[row * idx_cap + i];
            if (p >= 0 && p < Tcap)
                c = ((unsigned long long)keys[row * Tcap + p] << 32) | (0xFFFFFFFFu - (uint32_t)(p + pos_offset));
        }
        cand[row * budget + i] = c;
    }
}

// The global top-B of every rank's candidates, per (sequence, query head):
// one CTA finds the budget-th largest composite with three radix passes over
// the score keys (11/11/10 bits) and takes the ties on it by position, then
// dilates the Top set by +-nbr, clips it to C = [sink, T - window), and writes
// the global index list and count and this shard's attended-row bitmap: the
// sink, window and selected positions in [shard_begin, shard_begin +
// shard_len) ∩ [0, T), in local coordinates.
__global__ void __launch_bounds__(kFinThreads)
merge_candidates_kernel(const unsigned long long *__restrict__ cand, int n_ranks, int budget, int B, int Hq,
                        const int32_t *__restrict__ ctx_len, int Tcap, int Wg, int sink, int window, int nbr,
                        int32_t *__restrict__ idx, int idx_cap, int32_t *__restrict__ count, int shard_begin,
                        int shard_len, int Wl, uint32_t *__restrict__ local_bits, uint32_t *__restrict__ flags) {
    extern __shared__ uint32_t msm[];
    uint32_t *top_s = msm;        // [Wg]
    uint32_t *tie_s = msm + Wg;   // [Wg]
    __shared__ uint32_t hist[kBins2];
    __shared__ int scratch[kFinThreads / 32 + 3];
    const int tid = threadIdx.x;
    const int h = blockIdx.x, b = blockIdx.y;
    const size_t row = (size_t)b * Hq + h;
    for (int w = tid; w < Wg; w += kFinThreads) {
        top_s[w] = 0u;
        tie_s[w] = 0u;
    }
    griddep_wait();
    griddep_launch_dependents();
    const int T = clamp_ctx(ctx_len[b], Tcap, flags, tid == 0 && h == 0 && b == 0);
    const int lo = sink, hi = T - window;
    const int n = n_ranks * budget;
    auto cand_at = [&](int i) -> unsigned long long {
        const int r = i / budget, k = i - r * budget;
        return __ldcg(cand + (((size_t)r * B + b) * Hq + h) * budget + k);
    };
    // valid candidates (non-zero composites whose position is a candidate of C)
    auto valid = [&](unsigned long long c, uint32_t *pos) {
        const uint32_t p = 0xFFFFFFFFu - (uint32_t)c;
        *pos = p;
        return c != 0ull && (int)p >= lo && (int)p < hi;
    };
    int mine = 0;
    for (int i = tid; i < n; i += kFinThreads) {
        uint32_t p;
        mine += valid(cand_at(i), &p) ? 1 : 0;
    }
    int n_valid;
    (void)block_excl_scan<kFinThreads>(mine, scratch, &n_valid);
    __syncthreads();
    if (n_valid <= budget) {
        for (int i = tid; i < n; i += kFinThreads) {
            uint32_t p;
            if (valid(cand_at(i), &p)) atomicOr(&top_s[p >> 5], 1u << (p & 31));
        }
    } else {
        // the budget-th largest key: 11 + 11 + 10 bits, each pass over the
        // candidates whose higher digits match the ones fixed so far
        uint32_t need = (uint32_t)budget, prefix = 0u;
        int fixed = 0;
#pragma unroll 1
        for (int pass = 0; pass < 3; ++pass) {
            const int dw = pass < 2 ? 11 : 10;
            const int nb = 1 << dw;
            const int shift = 32 - fixed - dw;
            for (int i = tid; i < nb; i += kFinThreads) hist[i] = 0u;
            __syncthreads();
            for (int i = tid; i < n; i += kFinThreads) {
                uint32_t p;
                const unsigned long long c = cand_at(i);
                const uint32_t key = (uint32_t)(c >> 32);
                if (valid(c, &p) && (fixed == 0 || (key >> (32 - fixed)) == prefix))
                    atomicAdd(&hist[(key >> shift) & (uint32_t)(nb - 1)], 1u);
            }
            __syncthreads();
            uint32_t rem;
            const uint32_t bin = (uint32_t)block_find_bin_desc<kFinThreads>(hist, nb, need, &rem, scratch, false);
            prefix = (prefix << dw) | bin;
            fixed += dw;
            need = rem;
        }
        const uint32_t tau = prefix;  // keys above it are Top; `need` of the keys equal to it, lowest positions first
        for (int i = tid; i < n; i += kFinThreads) {
            uint32_t p;
            const unsigned long long c = cand_at(i);
            if (!valid(c, &p)) continue;
            const uint32_t key = (uint32_t)(c >> 32);
            if (key > tau) atomicOr(&top_s[p >> 5], 1u << (p & 31));
            else if (key == tau) atomicOr(&tie_s[p >> 5], 1u << (p & 31));
        }
        __syncthreads();
        const int wpt = (Wg + kFinThreads - 1) / kFinThreads;
        const int wb = tid * wpt, we = min(wb + wpt, Wg);
        int tmine = 0;
        for (int w = wb; w < we; ++w) tmine += __popc(tie_s[w]);
        int tot;
        int before = block_excl_scan<kFinThreads>(tmine, scratch, &tot);
        for (int w = wb; w < we; ++w) {
            uint32_t t = tie_s[w];
            const int pc = __popc(t);
            uint32_t keep = 0u;
            if (before + pc <= (int)need) {
                keep = t;
            } else if (before < (int)need) {
                for (int k = 0; k < (int)need - before; ++k) {
                    const uint32_t low = t & (0u - t);
                    keep |= low;
                    t ^= low;
                }
            }
            top_s[w] |= keep;
            before += pc;
        }
    }
    __syncthreads();
    // neighbour fetch, clip to C, emit the global list; tie_s becomes I
    const int wpt = (Wg + kFinThreads - 1) / kFinThreads;
    const int wb = tid * wpt, we = min(wb + wpt, Wg);
    int emine = 0;
    for (int w = wb; w < we; ++w) {
        const uint32_t t = top_s[w];
        const uint32_t pv = w > 0 ? top_s[w - 1] : 0u, nx = w + 1 < Wg ? top_s[w + 1] : 0u;
        uint32_t e = t;
        for (int k = 1; k <= nbr; ++k) e |= (t << k) | (pv >> (32 - k)) | (t >> k) | (nx << (32 - k));
        e &= range_mask(w, lo, hi);
        emine += __popc(e);
        tie_s[w] = e;
    }
    int total;
    const int base = block_excl_scan<kFinThreads>(emine, scratch, &total);
    {
        const int lane = tid & 31;
        const uint32_t lt = (1u << lane) - 1u;
        int32_t *out = idx + row * (size_t)idx_cap;
        const int w_first = (tid - lane) * wpt, w_last = min(w_first + 32 * wpt, Wg);
        int run = __shfl_sync(kFull, base, 0);
        for (int w = w_first; w < w_last; ++w) {
            const uint32_t e = tie_s[w];
            const int slot = run + __popc(e & lt);
            if (((e >> lane) & 1u) && slot < idx_cap) out[slot] = (w << 5) + lane;
            run += __popc(e);
        }
    }
    if (tid == 0) {
        if (total > idx_cap) raise_flag(flags, TB_FLAG_IDX_OVERFLOW);
        count[row] = total < idx_cap ? total : idx_cap;
    }
    // this shard's attended rows: sink, window and I inside the shard (shard_begin % 32 == 0)
    const int w0 = shard_begin >> 5;
    const int shard_end = min(shard_begin + shard_len, T);
    for (int wl = tid; wl < Wl; wl += kFinThreads) {
        const int w = w0 + wl;
        const uint32_t sel = w < Wg ? tie_s[w] : 0u;
        const uint32_t kept = sel | range_mask(w, 0, min(sink, T)) | range_mask(w, max(sink, T - window), T);
        local_bits[row * Wl + wl] = kept & range_mask(w, shard_begin, shard_end);
    }
}

// ------------------------------------------------------ scores of a call

// The fp32 scores behind the last selection on a workspace, decoded from the
// order-preserving key image score_hist left there: candidates of C get their
// score, every other position NaN.
__global__ void __launch_bounds__(kThreads)
export_scores_kernel(const uint32_t *__restrict__ keys, const int32_t *__restrict__ ctx_len, int Hq, int Tcap,
                     int sink, int window, float *__restrict__ out) {
    const int p = blockIdx.x * kThreads + threadIdx.x;
    const int h = blockIdx.y, b = blockIdx.z;
    griddep_wait();
    griddep_launch_dependents();
    if (p >= Tcap) return;
    const int T = clamp_ctx(ctx_len[b], Tcap, nullptr, false);
    const size_t i = ((size_t)b * Hq + h) * Tcap + p;
    float v = __int_as_float(0x7fc00000);
    if (p >= sink && p < T - window) {
        const uint32_t k = keys[i];
        v = __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
    }
    out[i] = v;
}

template <int SEL, bool HIST>
cudaError_t launch_score_hist(const tb_dims &d, const float *qp, int64_t qp_stride, const uint16_t *Kp,
                              const int32_t *ctx_len, int32_t sink, int32_t window, int32_t budget, const SelWs &s,
                              cudaStream_t st) {
    // with the histogram: 2048 positions a CTA; keys only: chunks that make
    // the grid about two CTAs per SM, so every SM streams its share of K'
    int chunk = kHistChunk;
    if (!HIST) {
        const long long pairs = (long long)d.batch * d.n_kv_heads;
        const long long want = (long long)d.ctx_cap * pairs / (2LL * num_sms());
        chunk = (int)std::max(512LL, (want + 31) / 32 * 32);
    }
    dim3 grid_h((d.ctx_cap + chunk - 1) / chunk, d.n_kv_heads, d.batch);
    const int hsm = (kThreads / 32) * hist_ring(HIST) * 32 * d.d_proj * 2;  // the warps' rings of 32-row blocks
    cudaError_t e;
    if (d.d_proj == 32) {
        static std::atomic<int> smem_set32[kMaxDevices];
        if ((e = ensure_dynamic_smem((const void *)score_hist_kernel<32, SEL, HIST>, hsm, smem_set32)) != cudaSuccess)
            return e;
        return launch_pdl(score_hist_kernel<32, SEL, HIST>, grid_h, dim3(kThreads), hsm, st, qp, qp_stride, Kp,
                          ctx_len, d.n_q_heads, d.n_kv_heads, d.ctx_cap, sink, window, budget, chunk, s);
    }
    static std::atomic<int> smem_set16[kMaxDevices];
    if ((e = ensure_dynamic_smem((const void *)score_hist_kernel<16, SEL, HIST>, hsm, smem_set16)) != cudaSuccess)
        return e;
    return launch_pdl(score_hist_kernel<16, SEL, HIST>, grid_h, dim3(kThreads), hsm, st, qp, qp_stride, Kp, ctx_len,
                      d.n_q_heads, d.n_kv_heads, d.ctx_cap, sink, window, budget, chunk, s);
}

template <int SEL>
cudaError_t launch_sel(const tb_dims &d, const float *qp, int64_t qp_stride, const uint16_t *Kp,
                       const int32_t *ctx_len, int32_t sink, int32_t window, int32_t budget, int32_t nbr,
                       int32_t *idx, int32_t idx_cap, int32_t *count, uint32_t *sel_bits, void *ws,
                       cudaStream_t st) {
    const SelWs s = carve(d, ws);
    const int W = (d.ctx_cap + 31) / 32;
    const int nch = (d.ctx_cap + kChunk - 1) / kChunk;
    dim3 grid(nch, d.n_kv_heads, d.batch);
    cudaError_t e = launch_score_hist<SEL, true>(d, qp, qp_stride, Kp, ctx_len, sink, window, budget, s, st);
    if (e != cudaSuccess) return e;
    e = launch_pdl(mark_collect_kernel<SEL>, grid, dim3(kThreads), 0, st, ctx_len, d.n_q_heads, d.n_kv_heads,
                   d.ctx_cap, W, sink, window, s);
    if (e != cudaSuccess) return e;
    const size_t fsm = (size_t)kCandCache * 8 + (size_t)2 * W * 4 + (SEL == kSelInclusive ? kCandCache * 2 : 0);
    static std::atomic<int> smem_set[kMaxDevices];
    if (fsm > 48 * 1024) {
        e = ensure_dynamic_smem((const void *)finalize_kernel<SEL>, (int)fsm, smem_set);
        if (e != cudaSuccess) return e;
    }
    const int rows = sel_is_group(SEL) ? d.n_q_heads / kGroup : d.n_q_heads;
    return launch_pdl(finalize_kernel<SEL>, dim3(rows, d.batch), dim3(fin_threads<SEL>()), fsm, st, ctx_len, d.n_q_heads,
                      d.ctx_cap, W, sink, window, budget, nbr, idx, idx_cap, count, sel_bits, s);
}

}  // namespace

size_t select_ws_bytes(const tb_dims &d) { return carve_bytes(d); }

cudaError_t launch_score_select(const tb_dims &d, const float *qp, int64_t qp_stride,
                                const uint16_t *Kp, const int32_t *ctx_len, int32_t sink,
                                int32_t window, int32_t budget, int32_t nbr, int32_t group_reduce,
                                int32_t *idx, int32_t idx_cap, int32_t *count, uint32_t *sel_bits, void *ws,
                                cudaStream_t st) {
    const int algo = select_algorithm();
    if (group_reduce != 2 && algo != TB_SELECT_MULTI_KERNEL &&
        select_cluster_fits(d, group_reduce, algo == TB_SELECT_AUTO))
        return launch_score_select_cluster(d, qp, qp_stride, Kp, ctx_len, sink, window, budget, nbr, group_reduce,
                                           idx, idx_cap, count, sel_bits, ws, st);
    if (group_reduce == 0)
        return launch_sel<kSelGroupMax>(d, qp, qp_stride, Kp, ctx_len, sink, window, budget, nbr, idx, idx_cap,
                                        count, sel_bits, ws, st);
    if (group_reduce == 2)
        return launch_sel<kSelInclusive>(d, qp, qp_stride, Kp, ctx_len, sink, window, budget, nbr, idx, idx_cap,
                                         count, sel_bits, ws, st);
    if (group_reduce == 1)
        return launch_sel<kSelGroupSum>(d, qp, qp_stride, Kp, ctx_len, sink, window, budget, nbr, idx, idx_cap,
                                        count, sel_bits, ws, st);
    return launch_sel<kSelHead>(d, qp, qp_stride, Kp, ctx_len, sink, window, budget, nbr, idx, idx_cap, count,
                                sel_bits, ws, st);
}

cudaError_t launch_score_keys(const tb_dims &d, const float *qp, int64_t qp_stride, const uint16_t *Kp,
                              const int32_t *ctx_len, int32_t sink, int32_t window, int32_t group_reduce, void *ws,
                              cudaStream_t st) {
    const SelWs s = carve(d, ws);
    if (group_reduce == 0)
        return launch_score_hist<kSelGroupMax, false>(d, qp, qp_stride, Kp, ctx_len, sink, window, 1, s, st);
    if (group_reduce == 1)
        return launch_score_hist<kSelGroupSum, false>(d, qp, qp_stride, Kp, ctx_len, sink, window, 1, s, st);
    return launch_score_hist<kSelHead, false>(d, qp, qp_stride, Kp, ctx_len, sink, window, 1, s, st);
}

cudaError_t launch_export_scores(const tb_dims &d, const void *ws, const int32_t *ctx_len, int32_t sink,
                                 int32_t window, float *scores, cudaStream_t st) {
    const SelWs s = carve(d, const_cast<void *>(ws));
    dim3 grid((d.ctx_cap + kThreads - 1) / kThreads, d.n_q_heads, d.batch);
    return launch_pdl(export_scores_kernel, grid, dim3(kThreads), 0, st, (const uint32_t *)s.keys, ctx_len,
                      d.n_q_heads, d.ctx_cap, sink, window, scores);
}

cudaError_t launch_export_candidates(const tb_dims &d, const void *ws, const int32_t *idx, int32_t idx_cap,
                                     const int32_t *count, int32_t budget, int32_t pos_offset, uint64_t *cand,
                                     cudaStream_t st) {
    const SelWs s = carve(d, const_cast<void *>(ws));
    return launch_pdl(export_candidates_kernel, dim3(d.n_q_heads, d.batch), dim3(kThreads), 0, st,
                      (const uint32_t *)s.keys, idx, idx_cap, count, d.n_q_heads, d.ctx_cap, budget, pos_offset,
                      reinterpret_cast<unsigned long long *>(cand));
}

cudaError_t launch_merge_candidates(const tb_dims &d, const uint64_t *cand, int32_t n_ranks, int32_t budget,
                                    const int32_t *ctx_len, int32_t sink, int32_t window, int32_t nbr, int32_t *idx,
                                    int32_t idx_cap, int32_t *count, int32_t shard_begin, int32_t shard_len,
                                    int32_t local_cap, uint32_t *local_bits, uint32_t *flags, cudaStream_t st) {
    const int Wg = (d.ctx_cap + 31) / 32, Wl = (local_cap + 31) / 32;
    const size_t sm = (size_t)2 * Wg * 4;
    static std::atomic<int> smem_set[kMaxDevices];
    if (sm > 48 * 1024) {
        cudaError_t e = ensure_dynamic_smem((const void *)merge_candidates_kernel, (int)sm, smem_set);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(merge_candidates_kernel, dim3(d.n_q_heads, d.batch), dim3(kFinThreads), sm, st,
                      reinterpret_cast<const unsigned long long *>(cand), n_ranks, budget, d.batch, d.n_q_heads,
                      ctx_len, d.ctx_cap, Wg, sink, window, nbr, idx, idx_cap, count, shard_begin, shard_len, Wl,
                      local_bits, flags);
}

cudaError_t launch_select_bits(const tb_dims &d, const int32_t *idx, int32_t idx_cap,
                               const int32_t *count, uint32_t *sel_bits, cudaStream_t st) {
    const int W = (d.ctx_cap + 31) / 32;
    const size_t sm = (size_t)W * 4;
    static std::atomic<int> smem_set[kMaxDevices];
    if (sm > 48 * 1024) {
        cudaError_t e = ensure_dynamic_smem((const void *)bits_from_idx_kernel, (int)sm, smem_set);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(bits_from_idx_kernel, dim3(d.n_q_heads, d.batch), dim3(kFinThreads), sm, st, idx, idx_cap,
                      count, d.n_q_heads, d.ctx_cap, W, sel_bits);
}

}  // namespace tb
