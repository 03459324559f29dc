// Exact top-B selection on thread-block clusters: one cluster per (sequence,
// KV head) holds all of the group's scores on chip and selects in one kernel.
//
// TokenButler technical summary (gist.science), "Core architecture: scoring":
// predicted queries dotted with projected keys give per-token importance
// scores that drive a budgeted selection; "Inference strategy": the first S
// (sink) and last N (window) tokens are always kept, so the candidates are
// C = [S, T-N); "Optimisations: prediction interval and neighbour fetch": the
// selected tokens are expanded by their neighbours.
//
// The result is the one the multi-kernel path (score_hist, mark_collect,
// finalize) computes, bit for bit: the same scores, the B largest
// order-preserving keys with ties on the B-th taken in position order, dilated
// by +-nbr and clipped to C.  Only the route differs.  The scores come first,
// from score_hist's keys-only variant on every SM (scoring streams K', which
// wants all of them); then one cluster per (sequence, KV head) selects.  CTA r
// of a cluster of CS owns the positions [r*L, (r+1)*L), L a multiple of 32:
//   1. keys   the CTA loads the keys of its slice from the workspace (just
//             written, so from L2) into shared memory, a warp per 32-position
//             word, lane = position; a histogram of key bits 31..21 per head
//             is built on the way.  Every later step loops over these words
//             (compact code: the kernel is otherwise bound by instruction
//             fetch).
//   2. radix  three passes (key bits 31..21, 20..10, 9..0) fix the B-th
//             largest key tau and k, how many keys equal to it are taken.  In
//             each, a CTA histograms its keys that match the digits fixed so
//             far, the cluster meets at a barrier, and every CTA sums the
//             cluster's histograms over distributed shared memory: first per
//             group of 32 bins, then the 32 bins of the group that holds the
//             B-th key.  Every CTA finds the same digit.
//   3. ties   the last histogram's bin tau holds each CTA's count of keys
//             equal to tau, so every CTA knows how many of its own (and its
//             neighbours') ties are taken, lowest positions first.
//   4. dilate the Top bitmap is dilated by +-nbr and clipped to C.  The edge
//             words of the neighbouring slices are rebuilt from the keys their
//             CTAs publish, so no extra barrier is needed for them.
//   5. emit   each CTA writes its slice's bitmap words and, at the offset the
//             lower slices' counts give, its part of the sorted index list.
// The cluster barriers sit at the same points on every path of every CTA of
// a cluster (the mode below depends only on the sequence's length), and a CTA
// leaves only after a last barrier, so no CTA reads the shared memory of one
// that has exited.
#include <algorithm>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "select_common.cuh"

namespace tb {
namespace {

using namespace sel;

constexpr int kCThreads = 1024;       // 32 warps
constexpr int kCWarps = kCThreads / 32;
constexpr int kHistWords = 2048 + 64; // per head: up to 2048 bins, then up to 64 group sums
constexpr int kCDynMax = 227 * 1024 - 4096;
constexpr int kMaxCluster = 16;
constexpr int kMinAutoSlice = 512;    // the automatic route takes the cluster kernel from this slice length

template <int SEL>
__host__ __device__ constexpr int rows_per_group() { return sel_is_group(SEL) ? 1 : kGroup; }
// Longest slice: its keys (4 bytes per position and score row) take 128 KB.
template <int SEL>
__host__ __device__ constexpr int max_slice() { return sel_is_group(SEL) ? 32768 : 8192; }
// Sum of the word at `local` over the shared memory of cluster CTAs 0 .. cs-1
// (every read issued before the first is added).
__device__ __forceinline__ uint32_t cluster_sum(const uint32_t *local, int cs) {
    uint32_t v[kMaxCluster];
#pragma unroll
    for (int q = 0; q < kMaxCluster; ++q) v[q] = q < cs ? *dsmem_ptr(local, (uint32_t)q) : 0u;
    uint32_t s = 0;
#pragma unroll
    for (int q = 0; q < kMaxCluster; ++q) s += v[q];
    return s;
}

// The cluster's histogram of one digit: every CTA has built its own in
// `hist` (per head: bins at [0, nb), group sums at [2048, 2048 + nb/32)).
// Finds, per head, the digit that holds the need[h]-th largest key and
// updates prefix[h] / need[h].  Whole CTA; call after a cluster barrier
// that follows the histogram and its group sums.
template <int NH>
__device__ void cluster_find_digit(const uint32_t *hist, int nb, int dbits, int cs, uint32_t *gco,
                                   uint32_t *prefix, uint32_t *need) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ng = nb / 32;
    // 1. the cluster's group sums
    if (tid < NH * ng) {
        const int h = tid / ng, j = tid % ng;
        gco[h * 64 + j] = cluster_sum(hist + h * kHistWords + 2048 + j, cs);
    }
    __syncthreads();
    if (warp < NH) {
        const int h = warp;
        const uint32_t nd = need[h];
        // 2. the group that holds the nd-th largest key (groups from the top)
        const int gpl = ng / 32;  // groups per lane: 2 or 1
        uint32_t c[2] = {0u, 0u};
        uint32_t v = 0;
#pragma unroll
        for (int q = 0; q < 2; ++q)
            if (q < gpl) {
                c[q] = gco[h * 64 + ng - 1 - (lane * gpl + q)];
                v += c[q];
            }
        uint32_t incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += t;
        }
        const uint32_t excl = incl - v;
        const bool cross = excl < nd && nd <= incl;
        int grp = 0;
        uint32_t above = 0;
        if (cross) {
            // the first of the lane's groups whose running count reaches nd
            const bool first = gpl == 1 || excl + c[0] >= nd;
            grp = ng - 1 - (lane * gpl + (first ? 0 : 1));
            above = first ? excl : excl + c[0];
        }
        const unsigned m = __ballot_sync(kFull, cross);
        const int src = m ? __ffs(m) - 1 : 0;
        grp = __shfl_sync(kFull, grp, src);
        above = __shfl_sync(kFull, above, src);
        // 3. its 32 bins, from the top
        const int bin = grp * 32 + 31 - lane;
        const uint32_t bv = cluster_sum(hist + h * kHistWords + bin, cs);
        uint32_t bi = bv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(kFull, bi, o);
            if (lane >= o) bi += t;
        }
        const uint32_t be = above + bi - bv;
        const bool hit = be < nd && nd <= above + bi;
        const unsigned hm = __ballot_sync(kFull, hit);
        const int hsrc = hm ? __ffs(hm) - 1 : 0;
        if (lane == hsrc) {
            prefix[h] = (prefix[h] << dbits) | (uint32_t)bin;
            need[h] = nd - be;
        }
    }
    __syncthreads();
}

// Group sums of the first radix pass's histogram (per head, 2048 bins):
// hist[h][2048 + j] = sum of bins [32j, 32j + 32).  A thread adds 4 bins read
// as one 16-byte word (a warp reads 512 consecutive bytes), and the 8 threads
// of a group combine theirs by shuffles.  Whole CTA, after the histogram is
// complete.
template <int NH>
__device__ void group_sums(uint32_t *hist) {
    constexpr int kChunks = 2048 / 4;  // per head
    static_assert((NH * kChunks) % 32 == 0 && kCThreads % 32 == 0, "whole warps in every round");
    for (int i = threadIdx.x; i < NH * kChunks; i += kCThreads) {
        const int h = i / kChunks, c = i % kChunks;
        const uint4 v = *reinterpret_cast<const uint4 *>(hist + h * kHistWords + 4 * c);
        uint32_t s = v.x + v.y + v.z + v.w;
        s += __shfl_xor_sync(kFull, s, 1);
        s += __shfl_xor_sync(kFull, s, 2);
        s += __shfl_xor_sync(kFull, s, 4);
        if ((c & 7) == 0) hist[h * kHistWords + 2048 + c / 8] = s;
    }
}

template <int SEL>
__global__ void __launch_bounds__(kCThreads, 1)
sel_cluster_kernel(const int32_t *__restrict__ ctx_len, int Hq, int Tcap, int W, int L, int sink, int window,
                   int budget, int nbr, int32_t *__restrict__ idx, int idx_cap, int32_t *__restrict__ count,
                   uint32_t *__restrict__ sel_bits, const uint32_t *__restrict__ gkeys, uint32_t *__restrict__ flags) {
    constexpr int NH = rows_per_group<SEL>();
    constexpr int NOUT = sel_is_group(SEL) ? kGroup : 1;  // output rows per score row
    const int LW = L / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    const int g = blockIdx.y, b = blockIdx.z;
    const int cs = (int)gridDim.x;
    const uint32_t r = cluster_ctarank();
    const int s0 = (int)r * L;

    // dynamic shared memory: [keys] [radix pass 2 histogram] [histogram A] [Top] [aux] [word prefix]
    extern __shared__ __align__(128) uint8_t csm[];
    uint32_t *keys_s = reinterpret_cast<uint32_t *>(csm);  // [NH][L]
    uint32_t *histB = keys_s + (size_t)NH * L;
    uint32_t *histA = histB + NH * kHistWords;
    uint32_t *top_s = histA + NH * kHistWords;
    uint32_t *aux_s = top_s + NH * LW;
    uint32_t *wpre_s = aux_s + NH * LW;
    __shared__ uint32_t edge_s[2][NH][32];  // keys of this slice's first and last word
    __shared__ uint32_t gco[4 * 64];
    __shared__ uint32_t prefix[4], need[4], x_cnt[4], base_s[4], total_s[4], take_s[4], nb_top[2][4];
    __shared__ int scratch[kCThreads / 32 + 3];

    for (int i = tid; i < NH * kHistWords; i += kCThreads) {
        histA[i] = 0u;
        histB[i] = 0u;
    }
    if (tid < 4) x_cnt[tid] = 0u;
    __syncthreads();  // the histograms are zero before any thread counts into them
    griddep_wait();   // the keys come from the kernel before
    griddep_launch_dependents();
    const int T = clamp_ctx(ctx_len[b], Tcap, flags, tid == 0 && r == 0 && g == 0);
    const int lo = sink, hi = T - window;
    const int nC = hi > lo ? hi - lo : 0;
    const uint32_t mode = nC == 0 ? kModeEmpty : (nC <= budget ? kModeAll : kModeSelect);
    const int a = max(lo, s0), e = min(hi, s0 + L);  // this slice's part of C
    const size_t krow0 = (size_t)b * Hq + (size_t)g * kGroup;  // first workspace key row of the group

    // ---- 1. the slice's keys into shared memory, word wi of score row h at
    // keys_s[h * L + 32 wi + lane]; 0 marks a position outside C (no score
    // has key 0: score_key maps every float, NaNs included, to a key of at
    // least 0x007fffff)
    {
        // the thread's loads go out 8 at a time, each batch issued before
        // its first key is used
        constexpr int WPW = max_slice<SEL>() / 32 / kCWarps;  // words of a score row per warp, at most
        constexpr int NLD = NH * WPW, BATCH = 8;
        static_assert(NLD % BATCH == 0, "whole batches");
#pragma unroll
        for (int b0 = 0; b0 < NLD; b0 += BATCH) {
            uint32_t kv[BATCH];
#pragma unroll
            for (int i = 0; i < BATCH; ++i) {
                const int h = (b0 + i) / WPW, wi = warp + kCWarps * ((b0 + i) % WPW);
                const int p = s0 + 32 * wi + lane;
                kv[i] = (wi < LW && p >= a && p < e) ? __ldcg(gkeys + (krow0 + h) * Tcap + p) : 0u;
            }
#pragma unroll
            for (int i = 0; i < BATCH; ++i) {
                const int h = (b0 + i) / WPW, wi = warp + kCWarps * ((b0 + i) % WPW);
                if (wi < LW) {  // warp-uniform
                    const uint32_t k = kv[i];
                    keys_s[h * L + 32 * wi + lane] = k;
                    if (k != 0u) atomicAdd(&histA[h * kHistWords + (k >> 21)], 1u);
                    if (wi == 0) edge_s[0][h][lane] = k;
                    if (wi == LW - 1) edge_s[1][h][lane] = k;
                }
            }
        }
    }
    __syncthreads();

    // ---- 2. radix passes -------------------------------------------------------
    if (mode == kModeSelect) {
        if (tid < NH) {
            prefix[tid] = 0u;
            need[tid] = (uint32_t)budget;
        }
        group_sums<NH>(histA);
        cluster_sync();
        cluster_find_digit<NH>(histA, 2048, 11, cs, gco, prefix, need);
        // key bits 20..10 of the keys whose bits 31..21 are prefix (few: counted with atomics)
#pragma unroll 1
        for (int h = 0; h < NH; ++h) {
            const uint32_t pf = prefix[h];
#pragma unroll 4
            for (int i = tid; i < L; i += kCThreads) {
                const uint32_t k = keys_s[h * L + i];
                if (k != 0u && (k >> 21) == pf) {
                    const uint32_t d = (k >> 10) & 0x7FFu;
                    atomicAdd(&histB[h * kHistWords + d], 1u);
                    atomicAdd(&histB[h * kHistWords + 2048 + (d >> 5)], 1u);
                }
            }
        }
        __syncthreads();
        cluster_sync();  // (also: every CTA is past its reads of histogram A)
        cluster_find_digit<NH>(histB, 2048, 11, cs, gco, prefix, need);
        for (int i = tid; i < NH * kHistWords; i += kCThreads) histA[i] = 0u;
        __syncthreads();
#pragma unroll 1
        for (int h = 0; h < NH; ++h) {
            const uint32_t pf = prefix[h];
#pragma unroll 4
            for (int i = tid; i < L; i += kCThreads) {
                const uint32_t k = keys_s[h * L + i];
                if (k != 0u && (k >> 10) == pf) {
                    const uint32_t d = k & 0x3FFu;
                    atomicAdd(&histA[h * kHistWords + d], 1u);
                    atomicAdd(&histA[h * kHistWords + 2048 + (d >> 5)], 1u);
                }
            }
        }
        __syncthreads();
        cluster_sync();
        cluster_find_digit<NH>(histA, 1024, 10, cs, gco, prefix, need);
        // now prefix[h] = tau, the B-th largest key, and need[h] = k
    }

    // ---- 3. Top and tie bitmaps of the slice ----------------------------------
    // (lane q keeps the ballots of the warp's q-th word and stores them after
    // the loop: one store per lane, no branch per word)
#pragma unroll 1
    for (int h = 0; h < NH; ++h) {
        const uint32_t tau = prefix[h];
        uint32_t my_top = 0u, my_tie = 0u;
        int q = 0;
#pragma unroll 2
        for (int wi = warp; wi < LW; wi += kCWarps, ++q) {
            const uint32_t k = keys_s[h * L + 32 * wi + lane];
            const bool v = k != 0u;
            bool gt = false, eq = false;
            if (mode == kModeSelect) {
                gt = v && k > tau;
                eq = v && k == tau;
            } else if (mode == kModeAll) {
                gt = v;
            }
            const uint32_t tb = __ballot_sync(kFull, gt), eb = __ballot_sync(kFull, eq);
            my_top = lane == q ? tb : my_top;
            my_tie = lane == q ? eb : my_tie;
        }
        const int wi = warp + kCWarps * lane;
        if (lane < q && wi < LW) {
            top_s[h * LW + wi] = my_top;
            aux_s[h * LW + wi] = my_tie;
        }
    }
    __syncthreads();
    if (mode == kModeSelect) {
        // bin tau & 1023 of each CTA's last histogram counts its keys equal
        // to tau: the ties each slice takes, in slice order, lowest first
        if (warp < NH) {
            const int h = warp;
            const uint32_t tau = prefix[h], k = need[h];
            const uint32_t t = lane < cs ? ld_dsmem(&histA[h * kHistWords + (tau & 0x3FFu)], (uint32_t)lane) : 0u;
            uint32_t incl = t;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t u = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += u;
            }
            const uint32_t before = incl - t;
            const uint32_t take = before >= k ? 0u : min(k - before, t);
            const uint32_t take_me = __shfl_sync(kFull, take, (int)r);
            const uint32_t take_prev = __shfl_sync(kFull, take, r > 0 ? (int)r - 1 : 0);
            const uint32_t ties_prev = __shfl_sync(kFull, t, r > 0 ? (int)r - 1 : 0);
            const uint32_t take_next = __shfl_sync(kFull, take, (int)r + 1 < cs ? (int)r + 1 : 0);
            // the neighbours' edge words, from the keys they published
            auto lowest = [](uint32_t m, int n) {  // the n lowest set bits of m
                uint32_t kept = 0u;
                for (int q = 0; q < n && m; ++q) {
                    const uint32_t low = m & (0u - m);
                    kept |= low;
                    m ^= low;
                }
                return kept;
            };
            uint32_t prev_top = 0u, next_top = 0u;
            if (r > 0) {
                const uint32_t pk = ld_dsmem(&edge_s[1][h][lane], r - 1);
                const int pp = s0 - 32 + lane;
                const bool ic = pp >= lo && pp < hi;
                const uint32_t gt = __ballot_sync(kFull, ic && pk > tau), eq = __ballot_sync(kFull, ic && pk == tau);
                const int n = (int)take_prev - ((int)ties_prev - __popc(eq));
                prev_top = gt | lowest(eq, n);
            }
            if ((int)r + 1 < cs) {
                const uint32_t nk = ld_dsmem(&edge_s[0][h][lane], r + 1);
                const int np = s0 + L + lane;
                const bool ic = np >= lo && np < hi;
                const uint32_t gt = __ballot_sync(kFull, ic && nk > tau), eq = __ballot_sync(kFull, ic && nk == tau);
                next_top = gt | lowest(eq, (int)take_next);
            }
            if (lane == 0) {
                take_s[h] = take_me;
                nb_top[0][h] = prev_top;
                nb_top[1][h] = next_top;
            }
        }
    } else if (tid < NH) {
        // all of C or nothing: the neighbours' edge words follow from C alone
        const int h = tid;
        take_s[h] = 0u;
        nb_top[0][h] = (mode == kModeAll && r > 0) ? range_mask((s0 >> 5) - 1, lo, hi) : 0u;
        nb_top[1][h] = (mode == kModeAll && (int)r + 1 < cs) ? range_mask((s0 + L) >> 5, lo, hi) : 0u;
    }
    __syncthreads();
    if (mode == kModeSelect && warp < NH) {
        // this slice's share of the ties, lowest positions first
        const int h = warp;
        const int take = (int)take_s[h];
        int run = 0;
        for (int w0 = 0; w0 < LW && run < take; w0 += 32) {
            const int wi = w0 + lane;
            uint32_t t = wi < LW ? aux_s[h * LW + wi] : 0u;
            const int pc = __popc(t);
            int incl = pc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += v;
            }
            const int bef = run + incl - pc;
            uint32_t keep = 0u;
            if (bef + pc <= take) {
                keep = t;
            } else if (bef < take) {
                for (int q = 0; q < take - bef; ++q) {
                    const uint32_t low = t & (0u - t);
                    keep |= low;
                    t ^= low;
                }
            }
            if (wi < LW) top_s[h * LW + wi] |= keep;
            run += __shfl_sync(kFull, incl, 31);
        }
    }
    __syncthreads();

    // ---- 4. neighbour fetch, clip to C, per-word counts -----------------------
#pragma unroll
    for (int h = 0; h < NH; ++h) {
        uint32_t c = 0;
        for (int wi = tid; wi < LW; wi += kCThreads) {
            const int gw = (int)r * LW + wi;
            const uint32_t t = top_s[h * LW + wi];
            const uint32_t pv = wi > 0 ? top_s[h * LW + wi - 1] : nb_top[0][h];
            const uint32_t nx = wi + 1 < LW ? top_s[h * LW + wi + 1] : nb_top[1][h];
            uint32_t ev = t;
            for (int k = 1; k <= nbr; ++k) ev |= (t << k) | (pv >> (32 - k)) | (t >> k) | (nx << (32 - k));
            ev &= range_mask(gw, lo, hi);
            aux_s[h * LW + wi] = ev;
            if (gw < W) {
#pragma unroll
                for (int o = 0; o < NOUT; ++o) sel_bits[(krow0 + h + o) * W + gw] = ev;
            }
            c += __popc(ev);
        }
        c = __reduce_add_sync(kFull, c);
        if (lane == 0 && c) atomicAdd(&x_cnt[h], c);
    }
    __syncthreads();
    {
        // exclusive prefix of the counts over the words, heads one after another
        const int ni = NH * LW;
        const int ipt = (ni + kCThreads - 1) / kCThreads;
        const int ib = min(tid * ipt, ni), ie = min(ib + ipt, ni);
        int mine = 0;
        for (int f = ib; f < ie; ++f) mine += __popc(aux_s[f]);
        int tot;
        int run = block_excl_scan<kCThreads>(mine, scratch, &tot);
        for (int f = ib; f < ie; ++f) {
            wpre_s[f] = (uint32_t)run;
            run += __popc(aux_s[f]);
        }
    }

    // ---- 5. offsets from the lower slices, then the sorted index list ---------
    cluster_sync();
    if (warp < NH) {
        const uint32_t c = lane < cs ? ld_dsmem(&x_cnt[warp], (uint32_t)lane) : 0u;
        const uint32_t below = __reduce_add_sync(kFull, lane < (int)r ? c : 0u);
        const uint32_t all = __reduce_add_sync(kFull, c);
        if (lane == 0) {
            base_s[warp] = below;
            total_s[warp] = all;
        }
    }
    cluster_arrive();  // this CTA reads no other CTA's shared memory from here on
    __syncthreads();
    {
        uint32_t hstart = 0;  // this CTA's selected positions of the heads before h
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            const uint32_t base = base_s[h];
#pragma unroll 4
            for (int wi = warp; wi < LW; wi += kCWarps) {
                const uint32_t ev = aux_s[h * LW + wi];
                const uint32_t slot = base + (wpre_s[h * LW + wi] - hstart) + __popc(ev & lt);
                if (((ev >> lane) & 1u) && slot < (uint32_t)idx_cap) {
                    const int p = ((int)r * LW + wi) * 32 + lane;
#pragma unroll
                    for (int o = 0; o < NOUT; ++o) idx[(krow0 + h + o) * (size_t)idx_cap + slot] = p;
                }
            }
            hstart += x_cnt[h];
        }
    }
    if (r == 0 && tid < NH) {
        const uint32_t total = total_s[tid];
        if (total > (uint32_t)idx_cap) raise_flag(flags, TB_FLAG_IDX_OVERFLOW);
#pragma unroll
        for (int o = 0; o < NOUT; ++o) count[krow0 + tid + o] = total < (uint32_t)idx_cap ? (int)total : idx_cap;
    }
    cluster_wait();
}

// ---------------------------------------------------------------- host side

struct Plan {
    int cs = 0, L = 0, waves = 0;
    size_t smem = 0;
};

template <int SEL>
size_t plan_smem(int L) {
    constexpr int NH = rows_per_group<SEL>();
    return (size_t)NH * L * 4 + (size_t)2 * NH * kHistWords * 4 + (size_t)3 * NH * (L / 32) * 4;
}

// How many clusters of each size 1..16 the device holds at once (one CTA per
// SM at the largest shared-memory size), queried once per device; nullptr
// when the kernel cannot be set up.
template <int SEL>
const int *active_clusters() {
    static std::atomic<int> state[kMaxDevices];  // 0 unknown, 1 ready, -1 unusable
    static int table[kMaxDevices][kMaxCluster + 1];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    int st = state[dev].load(std::memory_order_acquire);
    if (st == 0) {
        std::lock_guard<std::mutex> lock(mu);
        st = state[dev].load(std::memory_order_relaxed);
        if (st == 0) {
            const void *fn = (const void *)sel_cluster_kernel<SEL>;
            static std::atomic<int> smem_set[kMaxDevices];
            const int smem = (int)plan_smem<SEL>(max_slice<SEL>());
            st = -1;
            if (ensure_dynamic_smem(fn, smem, smem_set) == cudaSuccess &&
                cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
                st = 1;
                for (int cs = 1; cs <= kMaxCluster; ++cs) {
                    cudaLaunchConfig_t cfg = {};
                    cfg.gridDim = dim3(cs, 1, 1);
                    cfg.blockDim = dim3(kCThreads);
                    cfg.dynamicSmemBytes = smem;
                    cudaLaunchAttribute attr[1];
                    attr[0].id = cudaLaunchAttributeClusterDimension;
                    attr[0].val.clusterDim.x = (unsigned)cs;
                    attr[0].val.clusterDim.y = 1;
                    attr[0].val.clusterDim.z = 1;
                    cfg.attrs = attr;
                    cfg.numAttrs = 1;
                    int n = 0;
                    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) n = 0;
                    table[dev][cs] = n;
                }
            }
            (void)cudaGetLastError();
            state[dev].store(st, std::memory_order_release);
        }
    }
    return st > 0 ? table[dev] : nullptr;
}

// Cluster size and slice length for dims `d`: the size that minimises waves x
// slice length (the time of a latency-bound cluster grows with its slice),
// larger clusters on ties; cs = 0 when no size holds a (sequence, KV head).
template <int SEL>
Plan make_plan(const tb_dims &d) {
    Plan p;
    const int *act = active_clusters<SEL>();
    if (!act) return p;
    const int Tcap = d.ctx_cap;
    const long long pairs = (long long)d.batch * d.n_kv_heads;
    long long best = -1;
    for (int cs = 1; cs <= kMaxCluster; ++cs) {
        const int L = ((Tcap + cs - 1) / cs + 31) / 32 * 32;
        const int used = (Tcap + L - 1) / L;  // CTAs that own positions
        if (L > max_slice<SEL>() || act[used] < 1 || plan_smem<SEL>(L) > (size_t)kCDynMax) continue;
        const long long cost = (pairs + act[used] - 1) / act[used] * (long long)L;
        if (best < 0 || cost < best || (cost == best && used > p.cs)) {
            best = cost;
            p.cs = used;
            p.L = L;
            p.waves = (int)((pairs + act[used] - 1) / act[used]);
            p.smem = plan_smem<SEL>(L);
        }
    }
    return p;
}

template <int SEL>
cudaError_t launch_cluster(const tb_dims &d, const Plan &p, const float *qp, int64_t qp_stride, const uint16_t *Kp,
                           const int32_t *ctx_len, int32_t sink, int32_t window, int32_t budget, int32_t nbr,
                           int32_t *idx, int32_t idx_cap, int32_t *count, uint32_t *sel_bits, void *ws,
                           cudaStream_t st, int32_t group_reduce) {
    cudaError_t e = launch_score_keys(d, qp, qp_stride, Kp, ctx_len, sink, window, group_reduce, ws, st);
    if (e != cudaSuccess) return e;
    const SelWs s = carve(d, ws);
    const int W = (d.ctx_cap + 31) / 32;
    return launch_pdl_cluster(sel_cluster_kernel<SEL>, dim3(p.cs, d.n_kv_heads, d.batch), dim3(kCThreads), p.cs,
                              p.smem, st, ctx_len, d.n_q_heads, d.ctx_cap, W, p.L, sink, window, budget, nbr, idx,
                              idx_cap, count, sel_bits, (const uint32_t *)s.keys, s.flags);
}

template <int SEL>
Plan plan_for(const tb_dims &d) {
    return make_plan<SEL>(d);
}

}  // namespace

bool select_cluster_fits(const tb_dims &d, int32_t group_reduce, bool one_wave) {
    Plan p;
    switch (group_reduce) {
        case -1: p = plan_for<kSelHead>(d); break;
        case 0: p = plan_for<kSelGroupMax>(d); break;
        case 1: p = plan_for<kSelGroupSum>(d); break;
        default: return false;
    }
    // (shorter slices leave the cluster kernel's fixed latency, ~30 barrier
    // and exchange steps, larger than the multi-kernel path's whole cost)
    return p.cs > 0 && (!one_wave || (p.waves == 1 && p.L >= kMinAutoSlice));
}

cudaError_t launch_score_select_cluster(const tb_dims &d, const float *qp, int64_t qp_stride, const uint16_t *Kp,
                                        const int32_t *ctx_len, int32_t sink, int32_t window, int32_t budget,
                                        int32_t nbr, int32_t group_reduce, int32_t *idx, int32_t idx_cap,
                                        int32_t *count, uint32_t *sel_bits, void *ws, cudaStream_t st) {
    auto go = [&](auto sel_tag) -> cudaError_t {
        constexpr int SEL = decltype(sel_tag)::value;
        const Plan p = plan_for<SEL>(d);
        if (p.cs == 0) return cudaErrorNotSupported;
        return launch_cluster<SEL>(d, p, qp, qp_stride, Kp, ctx_len, sink, window, budget, nbr, idx, idx_cap, count,
                                   sel_bits, ws, st, group_reduce);
    };
    switch (group_reduce) {
        case -1: return go(std::integral_constant<int, kSelHead>());
        case 0: return go(std::integral_constant<int, kSelGroupMax>());
        case 1: return go(std::integral_constant<int, kSelGroupSum>());
        default: return cudaErrorNotSupported;
    }
}

}  // namespace tb
