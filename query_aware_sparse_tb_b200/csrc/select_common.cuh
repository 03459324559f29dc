// Constants, workspace layout and block-level helpers shared by the
// selection kernels (select.cu: the multi-kernel path; select_cluster.cu:
// the one-kernel cluster path).  Not part of the ABI.
#pragma once

#include "common.cuh"

namespace tb {
namespace sel {

constexpr int kGroup = 4;
constexpr int kChunk = 2048;          // positions per CTA of mark_collect (one wave at 64K)
constexpr int kHistChunk = 2048;      // positions per CTA of score_hist (one wave at 64K)
// 32-row blocks in each score_hist warp's ring: 3 in flight beside the
// histogram, 5 when the kernel only writes keys (two CTAs per SM either way)
__host__ __device__ constexpr int hist_ring(bool hist) { return hist ? 4 : 6; }
constexpr int kThreads = 256;
constexpr int kBins1 = 2048;          // key bits 31..21
constexpr int kBins2 = 2048;          // key bits 20..10
constexpr int kBins3 = 1024;          // key bits 9..0
constexpr int kFinThreads = 1024;
constexpr int kCandCache = 8192;      // candidates staged in shared memory by finalize
constexpr unsigned kFull = 0xffffffffu;

enum : uint32_t { kModeEmpty = 0, kModeAll = 1, kModeSelect = 2 };

// What is selected: one set per query head, or one set per KV head (group)
// from the largest or the fp32 sum (heads in order) of the group's scores.
// A group's set is kept in the rows of its first head until finalize copies
// it to all 4 heads.
enum : int { kSelHead = 0, kSelGroupMax = 1, kSelGroupSum = 2, kSelInclusive = 3 };
// kSelInclusive: per query head, but the importance buffer itself holds at
// most B tokens (candidates in score order while the union of their
// neighbourhoods fits); its budget is at most kCandCache.
__host__ __device__ constexpr bool sel_is_group(int sel) { return sel == kSelGroupMax || sel == kSelGroupSum; }

struct HeadState {   // 8 words per (b, query head)
    uint32_t mode, b1, k_rem, cand_count, n_in_bin, pad[3];
};

struct SelWs {
    uint32_t *flags, *keys, *hist, *counters;
    HeadState *state;
    unsigned long long *cand;
    uint32_t *top;
};

inline SelWs carve(const tb_dims &d, void *ws) {
    uint8_t *p = static_cast<uint8_t *>(ws);
    const size_t rows = (size_t)d.batch * d.n_q_heads;
    SelWs s;
    size_t off = 0;
    s.flags = reinterpret_cast<uint32_t *>(p);
    off += kWsHeaderBytes;
    s.keys = reinterpret_cast<uint32_t *>(p + off);
    off += align_up(rows * d.ctx_cap * 4, 256);
    s.hist = reinterpret_cast<uint32_t *>(p + off);
    off += align_up(rows * kBins1 * 4, 256);
    s.state = reinterpret_cast<HeadState *>(p + off);
    off += align_up(rows * sizeof(HeadState), 256);
    s.counters = reinterpret_cast<uint32_t *>(p + off);
    off += align_up((size_t)d.batch * d.n_kv_heads * 4, 256);
    s.cand = reinterpret_cast<unsigned long long *>(p + off);
    off += align_up(rows * d.ctx_cap * 8, 256);
    s.top = reinterpret_cast<uint32_t *>(p + off);
    return s;
}

inline size_t carve_bytes(const tb_dims &d) {
    const size_t rows = (size_t)d.batch * d.n_q_heads;
    const size_t W = (d.ctx_cap + 31) / 32;
    return kWsHeaderBytes + align_up(rows * d.ctx_cap * 4, 256) + align_up(rows * kBins1 * 4, 256) +
           align_up(rows * sizeof(HeadState), 256) + align_up((size_t)d.batch * d.n_kv_heads * 4, 256) +
           align_up(rows * d.ctx_cap * 8, 256) + align_up(rows * W * 4, 256);
}

// Exclusive prefix sum over the block (NT threads, in thread order); *total
// gets the sum.  `scratch` holds NT/32 + 1 ints.  All threads must call.
template <int NT>
__device__ int block_excl_scan(int v, int *scratch, int *total) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < NW ? scratch[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(kFull, wi, o);
            if (lane >= o) wi += t;
        }
        if (lane < NW) scratch[lane] = wi - w;
        if (lane == NW - 1) scratch[NW] = wi;
    }
    __syncthreads();
    const int res = scratch[warp] + incl - v;
    *total = scratch[NW];
    __syncthreads();
    return res;
}

// The bin that holds the `need`-th largest key of a histogram (bins in key
// order), searched from the top by the whole block: thread t owns the t-th
// group of bins counted from the top, a block scan gives every thread the
// count above its group, and the one thread whose group crosses `need` walks
// it.  Returns the bin; *rem = how many keys of that bin are still needed.
// `hist` may be global (read through L2) or shared; `scratch` holds NT/32 + 3
// ints.  All threads must call; nbins is a multiple of NT.
template <int NT>
__device__ int block_find_bin_desc(const uint32_t *hist, int nbins, uint32_t need, uint32_t *rem,
                                   int *scratch, bool from_global) {
    const int per = nbins / NT;
    const int hi = nbins - threadIdx.x * per;  // this thread's bins are [hi - per, hi)
    int mine = 0;
    for (int j = 1; j <= per; ++j) mine += (int)(from_global ? __ldcg(hist + hi - j) : hist[hi - j]);
    int total;
    const int above = block_excl_scan<NT>(mine, scratch, &total);
    if ((uint32_t)above < need && need <= (uint32_t)(above + mine)) {
        uint32_t acc = (uint32_t)above;
        for (int j = 1; j <= per; ++j) {
            const uint32_t v = from_global ? __ldcg(hist + hi - j) : hist[hi - j];
            if (acc + v >= need) {
                scratch[NT / 32 + 1] = hi - j;
                scratch[NT / 32 + 2] = (int)(need - acc);
                break;
            }
            acc += v;
        }
    }
    __syncthreads();
    const int bin = scratch[NT / 32 + 1];
    *rem = (uint32_t)scratch[NT / 32 + 2];
    __syncthreads();
    return bin;
}

__device__ __forceinline__ uint32_t range_mask(int w, int lo, int hi) {
    if (hi <= lo) return 0u;
    const int start = max(lo - (w << 5), 0), end = min(hi - (w << 5), 32);
    if (end <= start) return 0u;
    const uint32_t upto = end == 32 ? 0xffffffffu : ((1u << end) - 1u);
    return upto & ~((1u << start) - 1u);
}

}  // namespace sel
}  // namespace tb
