// Decode attention over the kept rows of a GQA group: sparse (sink ∪ window ∪
// selected) and dense (all rows) share one kernel template.
//
// TokenButler technical summary (gist.science), "Inference strategy": the
// cache is split into a sink (first S tokens, always kept), a local window
// (last N tokens, always kept) and an importance buffer filled from the
// predicted scores; "Significance": the full cache stays resident and only the
// selected tokens are read, which is what relieves the memory-bandwidth
// bottleneck.  The attention itself is standard scaled dot-product attention
// restricted to those rows (fp32 logits, fp32 online softmax, fp32 sums).
//
// Work split: one CTA per (sequence b, KV head g, context slice), one CTA per
// SM.  Every kept (b, g, t) row crosses HBM once for the whole group of 4
// query heads.  Warp roles:
//   * 4 load warps build the slice's row list (sparse: union over the group's
//     heads of their selected bits, plus sink and window rows, each row
//     tagged with a 4-bit head mask; compacted just ahead of the tiles that
//     read it) and stream 128-row K and V tiles into a 3-stage shared-memory
//     ring with cp.async, in the 128-byte-swizzled layout the tensor cores
//     read;
//   * 2 MMA warps issue (one the S products, one the PV products), per tile, S^T = K Q^T (M = 128 rows, N = 16 with the
//     4 heads in columns 0..3) and O^T = V^T P^T (M = 128 head dims, N = 16:
//     columns 0..3 take the bf16 high parts of the softmax weights, 4..7 the
//     bf16 remainders, so the weights keep ~16 significant bits), both bf16
//     tcgen05.mma into fp32 TMEM accumulators;
//   * 4 softmax warps (thread = tile row, then thread = head dim) read the
//     logits from TMEM, keep the online-softmax state, write P to shared
//     memory and fold each tile's O^T into fp32 registers.
// The S product of tile i+1 overlaps the softmax of tile i, and the PV
// product of tile i overlaps the softmax of tile i+1.  The last CTA of each
// (b, g), found with an atomic ticket, never a wait, merges the slices'
// partial states into the fp32 output.
//
// Every mbarrier wait is bounded; a wait that runs out flags TB_FLAG_TIMEOUT,
// tells the other roles through shared memory, and every role leaves its loop
// (the roles agree before each named barrier, so none is left waiting there).
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace tb {
namespace {

constexpr int kGroup = 4;          // query heads per KV head
constexpr int kRows = 128;         // KV rows per tile (M of the S^T product)
constexpr int kStages = 3;
constexpr int kSub = 4096;         // positions per row list (sparse)
constexpr int kMaxSplits = 64;     // partial states merged per (sequence, KV head)
static_assert(TB_ATTN_PLAN_STRIDE == kMaxSplits + 1, "a plan row holds every cut");
constexpr int kPlanThreads = 1024;
constexpr int kN = 16;             // N of both products (padded)
constexpr int kRoleThreads = 128;  // threads of the softmax role and of the load role
constexpr int kThreads = 2 * kRoleThreads + 64;  // + an S-issue warp and a PV-issue warp
constexpr int kMergeThreads = 256;
constexpr uint32_t kTmemCols = 64;  // S^T x2 buffers, O^T x2 buffers, 16 columns each
constexpr unsigned kFull = 0xffffffffu;
constexpr float kLazy = 8.0f;
// named barrier ids (0 is __syncthreads)
constexpr uint32_t kBarLoad = 1, kBarMath = 2, kBarMath2 = 3;

// Shared memory map, offsets from the 1024-byte aligned base.
struct Smem {
    static constexpr int kHalf = kRows * 128;         // [128 rows][64 dims] bf16, swizzled
    static constexpr int kSlot = 2 * kHalf;           // one tensor tile, head dims 0..63 | 64..127
    static constexpr int kStage = 2 * kSlot;          // K tile, V tile
    static constexpr int kQ = kStages * kStage;       // Q operand: 2 dim halves x 16 rows x 128 B
    static constexpr int kP = kQ + 4096;              // P operands: 2 buffers x (2 row halves x 16 x 128 B)
    static constexpr int kMask = kP + 2 * 4096;       // head masks [kStages][kRows]
    static constexpr int kList = kMask + kStages * kRows;  // row list: (offset << 4) | mask, uint16
    static constexpr int kWsum = kList + kSub * 2;         // per-warp row counts of the list build
    static constexpr int kWords = kWsum + 64;              // staged words: 4 head masks (uint4) each
    static constexpr int kWoff = kWords + (kSub / 32) * 16; // staged words: first list slot, + end
    static constexpr int kBar = kWoff + (kSub / 32 + 4) * 4;
    static constexpr int kNumBars = 2 * kStages + 10;
    static constexpr int kMisc = kBar + kNumBars * 8;  // tmem base, abort, n_rows, meta, reductions
    static constexpr int kEnd = kMisc + 256;
    static constexpr int kBytes = kEnd + 1024;  // + alignment slack
    static_assert(kQ % 1024 == 0 && kP % 1024 == 0, "operand alignment");
    static_assert(kBar % 8 == 0, "mbarrier alignment");
};
static_assert(Smem::kBytes <= 227 * 1024, "shared memory");

// Misc area layout (int/float words)
constexpr int kMiscTmem = 0, kMiscAbort = 1, kMiscMeta = 4, kMiscRed = 8;  // red: 2 x 16 floats

// A bounded mbarrier wait that also gives up as soon as another role of the
// CTA has given up.  The thread sleeps in the barrier between checks.
__device__ __forceinline__ bool wait_role(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          uint32_t *flags) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > kWaitBudgetCycles) {
            raise_flag(flags, TB_FLAG_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
}

// Shared-memory store of 16 bits when `pred` is non-zero (predicated, no branch).
__device__ __forceinline__ void st_shared_u16_if(uint32_t addr, uint16_t v, uint32_t pred) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.u32 p, %2, 0;\n\t"
        "@p st.shared.u16 [%0], %1;\n\t}\n" ::"r"(addr),
        "h"(v), "r"(pred)
        : "memory");
}

// bits 0 .. n-1 set (n clamped to [0, 32])
__device__ __forceinline__ uint32_t bits_below(int n) {
    return n <= 0 ? 0u : n >= 32 ? 0xffffffffu : (1u << n) - 1u;
}

// byte offset of element (row r, 16-byte chunk c) in a [rows][64] bf16 half
// written with the 128-byte swizzle (1024-byte atoms of 8 rows)
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
    return (uint32_t)(r * 128 + (((c ^ r) & 7) << 4));
}

template <int D, bool SPARSE>
__global__ void __launch_bounds__(kThreads, 1)
attn_kernel(const uint16_t *__restrict__ Q, const uint16_t *__restrict__ K,
            const uint16_t *__restrict__ V, const int32_t *__restrict__ ctx_len,
            const uint32_t *__restrict__ sel_bits, int Hq, int Hkv, int Tcap, int W, int sink,
            int window, float qscale, int splits, float *__restrict__ part,
            uint32_t *__restrict__ counters, float *__restrict__ out, uint32_t *__restrict__ flags,
            int early_trigger, int prefetch, float *__restrict__ part_out, const int32_t *__restrict__ plan) {
    constexpr int CPR = D / 8;      // 16-byte chunks per row
    constexpr int RPI = 32 / CPR;   // rows per warp-wide copy instruction
    constexpr int kKSteps = D / 16; // MMA K steps of S^T
    // one partial state per head: O[D], M, L, 2 pad floats (16-byte aligned records)
    constexpr int kHS = D + 4;
    constexpr int kPartStride = kGroup * kHS;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_addr(sm);
    uint8_t *masks = sm + Smem::kMask;
    const uint16_t *list = reinterpret_cast<const uint16_t *>(sm + Smem::kList);
    const uint32_t list_s = sb + Smem::kList;
    volatile int *wsum = reinterpret_cast<volatile int *>(sm + Smem::kWsum);
    uint4 *words_s = reinterpret_cast<uint4 *>(sm + Smem::kWords);
    int *woff_s = reinterpret_cast<int *>(sm + Smem::kWoff);
    volatile int *misc = reinterpret_cast<volatile int *>(sm + Smem::kMisc);
    volatile int *abort_flag = misc + kMiscAbort;
    volatile int *meta = misc + kMiscMeta;
    float *red = reinterpret_cast<float *>(sm + Smem::kMisc) + kMiscRed;
    const uint32_t qbase = sb + Smem::kQ, pbase = sb + Smem::kP;
    auto bar = [&](int i) -> uint32_t { return sb + Smem::kBar + 8u * (uint32_t)i; };
    auto full = [&](int s) { return bar(s); };
    auto empty = [&](int s) { return bar(kStages + s); };
    auto s_done = [&](int q) { return bar(2 * kStages + q); };
    auto p_ready = [&](int q) { return bar(2 * kStages + 2 + q); };
    auto o_done = [&](int q) { return bar(2 * kStages + 4 + q); };
    auto o_free = [&](int q) { return bar(2 * kStages + 6 + q); };
    const uint32_t drain = bar(2 * kStages + 8);
    const uint32_t q_ready = bar(2 * kStages + 9);
    __shared__ int s_last;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.z, g = blockIdx.y, split = blockIdx.x;

    // ------------------------------------------------------------ set-up
    // (touches only this CTA's shared memory and TMEM, so under a programmatic
    // launch it overlaps the end of the previous kernel in the stream)
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full(s), kRoleThreads);
            mbar_init(empty(s), 1);
        }
        for (int q = 0; q < 2; ++q) {
            mbar_init(s_done(q), 1);
            mbar_init(p_ready(q), kRoleThreads);
            mbar_init(o_done(q), 1);
            mbar_init(o_free(q), kRoleThreads);
        }
        mbar_init(drain, 2);
        mbar_init(q_ready, kRoleThreads);
        misc[kMiscAbort] = 0;
        fence_mbar_init();
    }
    if (warp == 8) {  // the S-issue warp owns the TMEM allocation
        tmem_alloc(sb + Smem::kMisc + 4 * kMiscTmem, kTmemCols);
        tmem_relinquish();
    }
    // Without prefetch, every input and the workspace may be written by the
    // previous kernel: wait for it before any global access.  With prefetch,
    // the lengths, the selection words and the K/V rows below T-1 are not
    // written by it (the caller's contract), so the load warps start on them
    // at once; Q, row T-1, the output and the workspace wait for it.
    if (!prefetch) {
        griddep_wait();
        // a one-wave grid lets the next kernel's CTAs take the SMs it leaves
        // idle and the ones its CTAs free; a longer grid only once this CTA
        // is done
        if (early_trigger) griddep_launch_dependents();
    }

    const int T = clamp_ctx(ctx_len[b], Tcap, flags, tid == 0 && split == 0 && g == 0);
    const size_t slab = ((size_t)b * Hkv + g) * (size_t)Tcap;
    const uint16_t *Kb = K + slab * D;
    const uint16_t *Vb = V + slab * D;
    float *part_bg = part + (size_t)(b * Hkv + g) * splits * kPartStride;
    const int pt = tid - kRoleThreads, pw = warp - 4;
    const bool loader = warp >= 4 && warp < 8;
    const uint32_t *sbits = sel_bits + ((size_t)b * Hq + (size_t)g * kGroup) * W;
    const int hi_c = T - window;  // candidates are [sink, hi_c)

    // This CTA's slice [p_begin, p_end) of (b, g), cut at whole 32-position
    // selection words.  Without a plan: equal shares of the length (slice s
    // opens at the word that holds position s * T / splits); sparse and dense
    // use the same slices, so with every candidate selected they do identical
    // arithmetic.  With a plan (tb_attn_plan: word indices at which equal
    // shares of the kept rows begin, counted once per prediction): its cuts,
    // clamped to [0, T), the first slice opening at 0 and the last closing at
    // T.  (Counting the kept rows here, at every launch, cost more at the
    // start than the balance saved: 42.3 against 38.7 us per 64K launch.)
    int p_begin, p_end;
    if (plan == nullptr) {
        p_begin = (int)(((long long)split * T / splits) >> 5) << 5;
        p_end = split + 1 == splits ? T
                                    : max(p_begin, min((int)(((long long)(split + 1) * T / splits) >> 5) << 5, T));
    } else {
        // (a cut at or past T leaves an empty slice [T, T); every other cut is
        // a whole word below T, and neighbouring slices share their cut)
        const int32_t *pl = plan + (size_t)(b * Hkv + g) * TB_ATTN_PLAN_STRIDE;
        const int nw = (T + 31) >> 5;
        p_begin = split == 0 ? 0 : min(min(max(pl[split], 0), nw) << 5, T);
        p_end = split + 1 == splits ? T : max(p_begin, min(min(max(pl[split + 1], 0), nw) << 5, T));
    }
    const int ns = splits;  // every CTA writes a state, empty slices with M = -inf

    // sparse: load warp thread pt owns word pt (32 positions) of a sub-chunk;
    // the group's 4 selection words of the first sub-chunk are requested
    // before the set-up, those of the next one while the current is streamed
    uint32_t hw[kGroup] = {0u, 0u, 0u, 0u};
    // (words past the length are masked when the list is built)
    const int p_cap_end = min((p_end + 31) & ~31, Tcap);
    auto fetch_words = [&](int q0) {
        const int q1 = min(q0 + kSub, p_cap_end);
        if (q0 + 32 * pt < q1) {
#pragma unroll
            for (int h = 0; h < kGroup; ++h) hw[h] = __ldg(sbits + (size_t)h * W + (q0 >> 5) + pt);
        }
    };
    if (SPARSE && loader) fetch_words(p_begin);

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[kMiscTmem];

    float m_ref[kGroup], o_acc[kGroup], L[kGroup];
    bool math_fail = false;

    if (loader) {
        // ============================================================ loads
        int it = 0;
        bool fail = false;
        const int step = SPARSE ? kSub : max(p_end - p_begin, 1);
        for (int p0 = p_begin; p0 < p_end && !fail; p0 += step) {
            const int p1 = min(p0 + step, p_end);
            int n_rows = p1 - p0;
            if constexpr (SPARSE) {
                // union over the group of the kept positions of this word,
                // each tagged with its head mask (sink and window: all heads)
                const int p = p0 + 32 * pt;
                const uint32_t vmask = bits_below(p1 - p);
                const uint32_t forced = (bits_below(sink - p) | ~bits_below(hi_c - p)) & vmask;
                uint32_t keep[kGroup], U = 0u;  // keep[h]: positions head h attends to
#pragma unroll
                for (int h = 0; h < kGroup; ++h) {
                    keep[h] = (hw[h] & vmask) | forced;
                    U |= keep[h];
                }
                const int cnt = __popc(U);
                int incl = cnt;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int v = __shfl_up_sync(kFull, incl, o);
                    if (lane >= o) incl += v;
                }
                if (lane == 31) wsum[pw] = incl;
                bar_named(kBarLoad, kRoleThreads);
                int off = incl - cnt;
                for (int w = 0; w < pw; ++w) off += wsum[w];
                n_rows = wsum[0] + wsum[1] + wsum[2] + wsum[3];
                // stage the word; the list itself is written progressively,
                // just ahead of the tiles that read it (see compact_upto)
                words_s[pt] = make_uint4(keep[0], keep[1], keep[2], keep[3]);
                woff_s[pt] = off;
                if (pt == 0) woff_s[kSub / 32] = n_rows;
                fetch_words(p0 + step);
                bar_named(kBarLoad, kRoleThreads);
            }
            // sparse: list slots [0, woff_s[done]) are written once words
            // [0, done) are compacted; a round compacts 8 words, 2 per warp,
            // lane = bit, with predicated stores (no divergence)
            int done = 0;
            const int nwords = (p1 - p0 + 31) >> 5;
            auto compact_upto = [&](int rows_needed) {
                const uint32_t lt = (1u << lane) - 1u;
                while (done < nwords && woff_s[done] < rows_needed) {
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int wq = done + 2 * pw + j;
                        if (wq < nwords) {
                            const uint4 kq = words_s[wq];
                            const int o = woff_s[wq];
                            const uint32_t Uk = kq.x | kq.y | kq.z | kq.w;
                            const uint32_t mk = ((kq.x >> lane) & 1u) | (((kq.y >> lane) & 1u) << 1) |
                                                (((kq.z >> lane) & 1u) << 2) | (((kq.w >> lane) & 1u) << 3);
                            st_shared_u16_if(list_s + 2u * (uint32_t)(o + __popc(Uk & lt)),
                                             (uint16_t)(((wq * 32 + lane) << 4) | mk), (Uk >> lane) & 1u);
                        }
                    }
                    done += 8;
                }
            };
            const int n_tiles = (n_rows + kRows - 1) / kRows;
            for (int t = 0; t < n_tiles; ++t, ++it) {
                const int s = it % kStages;
                // row T-1 (always kept: the window's last row) is the last row
                // of the last tile of the CTA whose slice ends at T; the
                // previous kernel may be writing it
                if (prefetch && p1 == T && t == n_tiles - 1) griddep_wait();
                if constexpr (SPARSE) compact_upto(min((t + 1) * kRows, n_rows));
                bool ok = true;
                if (it >= kStages) ok = wait_role(empty(s), ((it / kStages) + 1) & 1, abort_flag, flags);
                if (bar_any(kBarLoad, kRoleThreads, !ok)) {
                    fail = true;
                    break;
                }
                const uint32_t kslot = sb + s * Smem::kStage, vslot = kslot + Smem::kSlot;
#pragma unroll
                for (int i = 0; i < CPR; ++i) {
                    const int r = pw * 32 + i * RPI + lane / CPR, c = lane % CPR;
                    const int gr = t * kRows + r;
                    const bool valid = gr < n_rows;
                    int pos = p0, mk = 0;
                    if (valid) {
                        if constexpr (SPARSE) {
                            const int e = list[gr];
                            pos = p0 + (e >> 4);
                            mk = e & 0xF;
                        } else {
                            pos = p0 + gr;
                            mk = 0xF;
                        }
                    }
                    const size_t off = (size_t)pos * D + c * 8;
                    const uint32_t so = (uint32_t)((c >> 3) * Smem::kHalf) + sw128_off(r, c);
                    cp_async16(kslot + so, Kb + off, valid);
                    cp_async16(vslot + so, Vb + off, valid);
                    if (c == 0) masks[s * kRows + r] = (uint8_t)mk;
                }
                if (pt == 0) meta[s] = 1;
                cp_async_mbar_arrive(full(s));
                mbar_arrive(full(s));
            }
            if constexpr (SPARSE) bar_named(kBarLoad, kRoleThreads);  // list and counts read before rebuilding
        }
        if (!fail) {  // end marker: a stage with no rows
            const int s = it % kStages;
            bool ok = true;
            if (it >= kStages) ok = wait_role(empty(s), ((it / kStages) + 1) & 1, abort_flag, flags);
            if (!bar_any(kBarLoad, kRoleThreads, !ok)) {
                if (pt == 0) meta[s] = 0;
                mbar_arrive(full(s));
            }
        }
        cp_async_wait_all();
    } else if (warp >= 8) {
        // ============================================================ MMA issue
        // warp 8 issues the S^T products, warp 9 the O^T products; each waits
        // on one barrier at a time.  S(i) needs tile i's rows and S buffer i&1
        // read by the softmax of tile i-2; PV(i) needs the softmax of tile i
        // and O buffer i&1 folded by the epilogue of tile i-2.  A tile's stage
        // is released by the commit after its PV product (the S product of
        // the tile has completed before its softmax could start).
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16_f32(kRows, kN);
            const uint32_t id_o = idesc_bf16_f32(128, kN) | (1u << 15);  // A (V^T) MN-major
            bool ok = wait_role(q_ready, 0, abort_flag, flags);
            for (int i = 0; ok; ++i) {
                const int s = i % kStages;
                ok = wait_role(full(s), (i / kStages) & 1, abort_flag, flags);
                if (!ok || meta[s] == 0) break;
                if (warp == 8) {
                    if (i >= 2) ok = wait_role(p_ready(i & 1), ((i >> 1) + 1) & 1, abort_flag, flags);
                    if (!ok) break;
                    fence_proxy_async_smem();
                    tc_fence_after();
                    const uint32_t kslot = sb + s * Smem::kStage;
                    const uint32_t d = tmem + (uint32_t)((i & 1) * kN);
#pragma unroll
                    for (int k = 0; k < kKSteps; ++k) {
                        const uint32_t ko = (uint32_t)((k >> 2) * Smem::kHalf + (k & 3) * 32);
                        const uint32_t qo = (uint32_t)((k >> 2) * 2048 + (k & 3) * 32);
                        umma_bf16(d, sw128_kmajor_desc(kslot + ko), sw128_kmajor_desc(qbase + qo), id_s, k > 0);
                    }
                    umma_commit(s_done(i & 1));
                } else {
                    ok = wait_role(p_ready(i & 1), (i >> 1) & 1, abort_flag, flags);
                    if (ok && i >= 2) ok = wait_role(o_free(i & 1), ((i >> 1) + 1) & 1, abort_flag, flags);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t vslot = sb + s * Smem::kStage + Smem::kSlot;
                    const uint32_t pb = pbase + (uint32_t)((i & 1) * 4096);
                    const uint32_t d = tmem + (uint32_t)(2 * kN + (i & 1) * kN);
#pragma unroll
                    for (int k = 0; k < kRows / 16; ++k) {
                        const uint32_t po = (uint32_t)((k >> 2) * 2048 + (k & 3) * 32);
                        umma_bf16(d, sw128_mnmajor_desc(vslot + k * 2048, Smem::kHalf), sw128_kmajor_desc(pb + po),
                                  id_o, k > 0);
                    }
                    umma_commit(o_done(i & 1));
                    umma_commit(empty(s));
                }
            }
            // every MMA of both issuers has finished before TMEM is released
            umma_commit(drain);
            mbar_wait_bounded(drain, 0, flags);
        }
        __syncwarp();
    } else {
        // ============================================================ softmax
        const int mt = tid;  // tile row, then head dim
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        {
            // P operands: rows 8..15 stay zero (shared memory only: before the wait)
            uint4 *pz = reinterpret_cast<uint4 *>(sm + Smem::kP);
            for (int e = mt; e < 2 * 4096 / 16; e += kRoleThreads) pz[e] = make_uint4(0u, 0u, 0u, 0u);
            if (prefetch) {
                griddep_wait();  // Q may come from the previous kernel
                if (early_trigger) griddep_launch_dependents();
            }
            // Q operand (K-major, 16 rows: the group's 4 query heads, then
            // zeros), one 16-byte chunk (8 dims) per load and per swizzled
            // store: all of a thread's loads are in flight at once
            const uint16_t *Qg = Q + ((size_t)b * Hq + (size_t)g * kGroup) * D;
            constexpr int kQChunks = kN * 16;  // 16 rows x (2 halves x 8 chunks of 8 dims)
            uint4 qv[kQChunks / kRoleThreads];
#pragma unroll
            for (int k = 0; k < kQChunks / kRoleThreads; ++k) {
                const int e = mt + k * kRoleThreads, n = e >> 4, c = e & 15;
                qv[k] = (n < kGroup && c * 8 < D) ? *reinterpret_cast<const uint4 *>(Qg + (size_t)n * D + c * 8)
                                                  : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int k = 0; k < kQChunks / kRoleThreads; ++k) {
                const int e = mt + k * kRoleThreads, n = e >> 4, c = e & 15;
                *reinterpret_cast<uint4 *>(sm + Smem::kQ + (c >> 3) * 2048 + (n >> 3) * 1024 + sw128_off(n & 7, c & 7)) =
                    qv[k];
            }
            fence_proxy_async_smem();
            mbar_arrive(q_ready);
        }
        float l_part[kGroup], mt0[kGroup], mt1[kGroup];
#pragma unroll
        for (int h = 0; h < kGroup; ++h) {
            m_ref[h] = -INFINITY;
            l_part[h] = 0.f;
            o_acc[h] = 0.f;
            mt0[h] = mt1[h] = -INFINITY;
        }
        // fold tile j's O^T (relative to that tile's references) into o_acc
        auto epilogue = [&](int j) -> bool {
            const bool ok = wait_role(o_done(j & 1), (j >> 1) & 1, abort_flag, flags);
            if (bar_any(kBarMath, kRoleThreads, !ok)) return false;
            tc_fence_after();
            float ov[8];
            tmem_ld8(tmem + lane_off + (uint32_t)(2 * kN + (j & 1) * kN), ov);
#pragma unroll
            for (int h = 0; h < kGroup; ++h) {
                const float mj = (j & 1) ? mt1[h] : mt0[h];
                const float f = (mj == m_ref[h]) ? 1.f : exp2f(mj - m_ref[h]);
                o_acc[h] = fmaf(ov[h] + ov[kGroup + h], f, o_acc[h]);
            }
            tc_fence_before();
            mbar_arrive(o_free(j & 1));
            return true;
        };
        int i = 0;
        for (;; ++i) {
            const int s = i % kStages;
            bool ok = wait_role(full(s), (i / kStages) & 1, abort_flag, flags);
            if (bar_any(kBarMath, kRoleThreads, !ok)) {
                math_fail = true;
                break;
            }
            if (meta[s] == 0) break;
            ok = wait_role(s_done(i & 1), (i >> 1) & 1, abort_flag, flags);
            if (bar_any(kBarMath, kRoleThreads, !ok)) {
                math_fail = true;
                break;
            }
            tc_fence_after();
            float sv[4];
            tmem_ld4(tmem + lane_off + (uint32_t)((i & 1) * kN), sv);
            const uint32_t mk = masks[s * kRows + mt];
            float t[kGroup];
            bool need = false;
#pragma unroll
            for (int h = 0; h < kGroup; ++h) {
                t[h] = ((mk >> h) & 1u) ? sv[h] * qscale : -INFINITY;
                need |= t[h] > m_ref[h] + kLazy;
            }
            // raise the per-head references (to the tile maximum) only when a
            // logit exceeds its reference by more than kLazy, so every weight
            // exp2(t - m_ref) stays <= 2^kLazy; the softmax is unchanged
            if (bar_any(kBarMath, kRoleThreads, need)) {
                float mx[kGroup];
#pragma unroll
                for (int h = 0; h < kGroup; ++h) {
                    mx[h] = t[h];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) mx[h] = fmaxf(mx[h], __shfl_xor_sync(kFull, mx[h], o));
                }
                if (lane == 0) {
#pragma unroll
                    for (int h = 0; h < kGroup; ++h) red[warp * kGroup + h] = mx[h];
                }
                bar_named(kBarMath2, kRoleThreads);
#pragma unroll
                for (int h = 0; h < kGroup; ++h) {
                    float mn = m_ref[h];
#pragma unroll
                    for (int w = 0; w < 4; ++w) mn = fmaxf(mn, red[w * kGroup + h]);
                    if (mn > m_ref[h]) {
                        const float alpha = exp2f(m_ref[h] - mn);  // 0 while m_ref is -inf
                        l_part[h] *= alpha;
                        o_acc[h] *= alpha;
                        m_ref[h] = mn;
                    }
                }
                bar_named(kBarMath2, kRoleThreads);  // red read by all before reuse
            }
            // weights as bf16 high part (N rows 0..3) + bf16 remainder (rows 4..7)
            uint8_t *pb = sm + Smem::kP + (i & 1) * 4096 + (mt >> 6) * 2048 + (mt & 7) * 2;
            const int rc = (mt & 63) >> 3;
#pragma unroll
            for (int h = 0; h < kGroup; ++h) {
                const float p = (t[h] == -INFINITY) ? 0.f : exp2f(t[h] - m_ref[h]);
                l_part[h] += p;
                const uint16_t hi = f32_to_bf16_rne(p);
                const uint16_t lo = f32_to_bf16_rne(p - __uint_as_float((uint32_t)hi << 16));
                *reinterpret_cast<uint16_t *>(pb + sw128_off(h, rc)) = hi;
                *reinterpret_cast<uint16_t *>(pb + sw128_off(kGroup + h, rc)) = lo;
                if (i & 1) mt1[h] = m_ref[h]; else mt0[h] = m_ref[h];
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(p_ready(i & 1));
            if (i >= 1 && !epilogue(i - 1)) {
                math_fail = true;
                break;
            }
        }
        if (!math_fail && i >= 1 && !epilogue(i - 1)) math_fail = true;

        // softmax sums over the 128 rows of the role
#pragma unroll
        for (int h = 0; h < kGroup; ++h) {
            float v = l_part[h];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
            if (lane == 0) red[16 + warp * kGroup + h] = v;
        }
        bar_named(kBarMath2, kRoleThreads);
#pragma unroll
        for (int h = 0; h < kGroup; ++h)
            L[h] = red[16 + h] + red[16 + kGroup + h] + red[16 + 2 * kGroup + h] + red[16 + 3 * kGroup + h];
        {
            float *pp = part_bg + (size_t)split * kPartStride;
            if (mt < D) {
#pragma unroll
                for (int h = 0; h < kGroup; ++h) pp[h * kHS + mt] = o_acc[h];
            }
            if (mt == 0) {
#pragma unroll
                for (int h = 0; h < kGroup; ++h) {
                    pp[h * kHS + D] = m_ref[h];
                    pp[h * kHS + D + 1] = L[h];
                }
            }
        }
    }

    // ---------------------------------------------------- release, ticket
    if (prefetch) griddep_wait();  // (roles that have not waited yet) before the workspace
    if (!early_trigger) griddep_launch_dependents();
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (tid == 0) {
        // one acquire-release ticket: its release publishes the CTA's partial
        // states (every thread's stores are ordered before it by the barrier
        // above), its acquire lets the last CTA read every other CTA's
        s_last = (atom_add_acq_rel_gpu(&counters[b * Hkv + g], 1u) == (unsigned)splits - 1u);
    }
    __syncthreads();
    if (!s_last) return;

    // ---------------------------------------------------- last CTA merges
    // One output group (head, 4 dims) per TPG threads; each thread loads its
    // share of the ns <= 64 partial states (one round for up to 32 splits),
    // scales them to the round's largest reference and sums, then the TPG
    // lanes combine with shuffles.
    constexpr int kGroups4 = kGroup * D / 4;
    constexpr int TPG = kMergeThreads / kGroups4;
    if (tid < kMergeThreads) {
        const int grp = tid / TPG, j = tid % TPG;
        const int h = grp / (D / 4), d4 = grp % (D / 4);
        const float *src = part_bg + h * kHS;
        float M = -INFINITY, Ls = 0.f;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        auto fold = [&](float m2, float l2, float4 o2) {
            if (m2 == -INFINITY) return;  // a slice with no kept row for this head
            const float Mn = fmaxf(M, m2);
            const float a = exp2f(M - Mn), c = exp2f(m2 - Mn);  // a = 0 while M is -inf
            o.x = fmaf(o.x, a, o2.x * c); o.y = fmaf(o.y, a, o2.y * c);
            o.z = fmaf(o.z, a, o2.z * c); o.w = fmaf(o.w, a, o2.w * c);
            Ls = fmaf(Ls, a, l2 * c);
            M = Mn;
        };
        constexpr int kU = 16;  // states loaded per round: one round for up to 32 splits
        for (int s0 = j; s0 < ns; s0 += kU * TPG) {
            float2 ml[kU];
            float4 v[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int s = s0 + u * TPG;
                if (s < ns) {
                    const float *rec = src + (size_t)s * kPartStride;
                    ml[u] = __ldcg(reinterpret_cast<const float2 *>(rec + D));
                    v[u] = __ldcg(reinterpret_cast<const float4 *>(rec + d4 * 4));
                } else {
                    ml[u] = make_float2(-INFINITY, 0.f);
                    v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            // the round's largest reference first, then every state scaled to
            // it independently (no chain of dependent rescales)
            float Mr = -INFINITY;
#pragma unroll
            for (int u = 0; u < kU; ++u) Mr = fmaxf(Mr, ml[u].x);
            if (Mr != -INFINITY) {
                float Lr = 0.f;
                float4 orr = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const float c = exp2f(ml[u].x - Mr);  // 0 for a slice with no kept row (-inf)
                    orr.x = fmaf(v[u].x, c, orr.x); orr.y = fmaf(v[u].y, c, orr.y);
                    orr.z = fmaf(v[u].z, c, orr.z); orr.w = fmaf(v[u].w, c, orr.w);
                    Lr = fmaf(ml[u].y, c, Lr);
                }
                fold(Mr, Lr, orr);
            }
        }
#pragma unroll
        for (int off = 1; off < TPG; off <<= 1) {
            const float m2 = __shfl_xor_sync(kFull, M, off), l2 = __shfl_xor_sync(kFull, Ls, off);
            float4 o2;
            o2.x = __shfl_xor_sync(kFull, o.x, off); o2.y = __shfl_xor_sync(kFull, o.y, off);
            o2.z = __shfl_xor_sync(kFull, o.z, off); o2.w = __shfl_xor_sync(kFull, o.w, off);
            fold(m2, l2, o2);
        }
        if (j == 0) {  // scalar stores: `out` is only required to be 4-byte aligned
            if (part_out) {
                // the unnormalised state (o relative to M, M, L) for a merge across shards
                float *dst = part_out + ((size_t)b * Hq + g * kGroup + h) * (D + 2);
                dst[d4 * 4] = o.x; dst[d4 * 4 + 1] = o.y; dst[d4 * 4 + 2] = o.z; dst[d4 * 4 + 3] = o.w;
                if (d4 == 0) {
                    dst[D] = M;
                    dst[D + 1] = Ls;
                }
            } else {
                const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
                float *dst = out + ((size_t)b * Hq + g * kGroup + h) * D + d4 * 4;
                dst[0] = o.x * inv; dst[1] = o.y * inv; dst[2] = o.z * inv; dst[3] = o.w * inv;
            }
        }
    }
    if (tid == 0) counters[b * Hkv + g] = 0u;  // leave the ticket zeroed for the next call
}

// out[b][h][:] = the merged state of n_parts unnormalised partial states
// parts[p][b][h] = (o[D], M, L) (log2 units): sum_p 2^(M_p - M*) o_p / sum_p 2^(M_p - M*) L_p
template <int D>
__global__ void __launch_bounds__(D)
combine_kernel(const float *__restrict__ parts, int n_parts, int rows, float *__restrict__ out) {
    const int r = blockIdx.x, d = threadIdx.x;
    griddep_wait();
    griddep_launch_dependents();
    float Mx = -INFINITY;
    for (int p = 0; p < n_parts; ++p) Mx = fmaxf(Mx, parts[((size_t)p * rows + r) * (D + 2) + D]);
    float o = 0.f, Ls = 0.f;
    if (Mx != -INFINITY) {
        for (int p = 0; p < n_parts; ++p) {
            const float *st = parts + ((size_t)p * rows + r) * (D + 2);
            const float m = st[D];
            if (m == -INFINITY) continue;  // a shard with no attended row of this head
            const float w = exp2f(m - Mx);
            o = fmaf(st[d], w, o);
            Ls = fmaf(st[D + 1], w, Ls);
        }
    }
    out[(size_t)r * D + d] = Ls > 0.f ? o / Ls : 0.f;
}

template <int D, bool SPARSE>
cudaError_t launch_t(const tb_dims &d, const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                     const int32_t *ctx_len, int32_t sink, int32_t window, const uint32_t *sel_bits,
                     float scale, float *out, void *ws, cudaStream_t st, float *part_out, const int32_t *plan) {
    static std::atomic<int> smem_set[kMaxDevices];
    cudaError_t e = ensure_dynamic_smem((const void *)attn_kernel<D, SPARSE>, Smem::kBytes, smem_set);
    if (e != cudaSuccess) return e;
    const int splits = attn_splits(d);
    uint8_t *w = static_cast<uint8_t *>(ws);
    uint32_t *flags = reinterpret_cast<uint32_t *>(w);
    uint32_t *counters = reinterpret_cast<uint32_t *>(w + kWsHeaderBytes);
    float *part = reinterpret_cast<float *>(
        w + kWsHeaderBytes + align_up((size_t)d.batch * d.n_kv_heads * 4, 256));
    const int W = (d.ctx_cap + 31) / 32;
    const float qscale = scale * 1.4426950408889634f;  // logits in log2 units for exp2
    // the launch may begin while the previous kernel in the stream finishes;
    // the kernel waits for it (griddep_wait) before its first global access
    const int early = (long long)splits * d.n_kv_heads * d.batch <= num_sms() ? 1 : 0;
    const int prefetch = attn_launch_mode() == TB_ATTN_PREFETCH_KV ? 1 : 0;
    return launch_pdl(attn_kernel<D, SPARSE>, dim3(splits, d.n_kv_heads, d.batch), dim3(kThreads), Smem::kBytes,
                      st, Q, K, V, ctx_len, sel_bits, d.n_q_heads, d.n_kv_heads, d.ctx_cap, W, sink, window, qscale,
                      splits, part, counters, out, flags, early, prefetch, part_out, plan);
}

// The plan of tb_attn_plan: one CTA per (b, g).  Word w of (b, g) weighs the
// kept rows it holds (the sink, the window and the group's selected positions,
// all below T); slice s of `splits` opens at the first word whose preceding
// weight reaches s/splits of the total.
__global__ void __launch_bounds__(kPlanThreads)
attn_plan_kernel(const uint32_t *__restrict__ sel_bits, const int32_t *__restrict__ ctx_len, int Hq, int Hkv,
                 int Tcap, int W, int sink, int window, int splits, int32_t *__restrict__ plan,
                 uint32_t *__restrict__ flags) {
    __shared__ int scratch[kPlanThreads / 32 + 1];
    __shared__ int s_total;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = blockIdx.x, b = blockIdx.y;
    griddep_wait();
    griddep_launch_dependents();
    const int T = clamp_ctx(ctx_len[b], Tcap, flags, false);
    const int nw = (T + 31) >> 5;
    const uint32_t *sbits = sel_bits + ((size_t)b * Hq + (size_t)g * kGroup) * W;
    const int lo_w = min(sink, T), hi_w = max(sink, T - window);
    auto weight = [&](int w) {
        uint32_t m = 0u;
#pragma unroll
        for (int h = 0; h < kGroup; ++h) m |= sbits[(size_t)h * W + w];
        const int base = w << 5;
        auto range = [&](int a, int e) -> uint32_t {  // bits of [a, e) in word w
            const int s0 = max(a - base, 0), s1 = min(e - base, 32);
            if (s1 <= s0) return 0u;
            return (s1 == 32 ? 0xffffffffu : ((1u << s1) - 1u)) & ~((1u << s0) - 1u);
        };
        m |= range(0, lo_w) | range(hi_w, T);
        m &= range(0, T);
        return __popc(m);
    };
    // contiguous runs of words per thread, an exclusive scan over the threads
    const int per = (nw + kPlanThreads - 1) / kPlanThreads;
    const int w0 = min(tid * per, nw), w1 = min(w0 + per, nw);
    int mine = 0;
    for (int w = w0; w < w1; ++w) mine += weight(w);
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int v = lane < kPlanThreads / 32 ? scratch[lane] : 0;
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += t;
        }
        if (lane < kPlanThreads / 32) scratch[lane] = x - v;
        if (lane == kPlanThreads / 32 - 1) s_total = x;
    }
    __syncthreads();
    const long long total = s_total;
    int32_t *out = plan + (size_t)(b * Hkv + g) * TB_ATTN_PLAN_STRIDE;
    // cut s (0 < s < splits) falls in the word where the running weight
    // crosses s * total / splits; the slice opens after that word
    int before = scratch[warp] + incl - mine;
    for (int w = w0; w < w1; ++w) {
        const int c = weight(w);
        for (int s = 1; s < splits; ++s) {
            const long long share = (long long)s * total;  // compared as weight * splits
            if (share > (long long)before * splits && share <= (long long)(before + c) * splits) out[s] = w + 1;
        }
        before += c;
    }
    if (tid == 0) {
        out[0] = 0;
        out[splits] = nw;
        if (total == 0)
            for (int s = 1; s < splits; ++s) out[s] = 0;
    }
}

}  // namespace

// CTAs per (sequence, KV head), one CTA per SM: the count s <= kMaxSplits that
// minimises waves(s) x (tiles per CTA + 2 tiles of pipeline fill), with the
// context capacity standing in for the (device-side) lengths.
int attn_splits(const tb_dims &d) {
    const long long slots = num_sms();
    const long long pairs = (long long)d.batch * d.n_kv_heads;
    const int max_useful = std::max(1, (d.ctx_cap + kRows - 1) / kRows);
    int best = 1;
    long long best_cost = -1;
    for (int s = 1; s <= std::min(kMaxSplits, max_useful); ++s) {
        const long long waves = (pairs * s + slots - 1) / slots;
        const long long tiles = ((long long)d.ctx_cap + (long long)s * kRows - 1) / ((long long)s * kRows);
        const long long cost = waves * (tiles + 2);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    return best;
}

size_t attn_ws_bytes(const tb_dims &d) {
    return kWsHeaderBytes + align_up((size_t)d.batch * d.n_kv_heads * 4, 256) +
           (size_t)d.batch * d.n_kv_heads * kMaxSplits * kGroup * (d.head_dim + 4) * 4;
}

cudaError_t launch_attn(const tb_dims &d, const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                        const int32_t *ctx_len, int32_t sink, int32_t window,
                        const uint32_t *sel_bits, bool sparse, float scale, float *out, void *ws,
                        cudaStream_t st, float *part_out, const int32_t *plan) {
    if (d.head_dim == 128) {
        return sparse ? launch_t<128, true>(d, Q, K, V, ctx_len, sink, window, sel_bits, scale, out, ws, st, part_out,
                                            plan)
                      : launch_t<128, false>(d, Q, K, V, ctx_len, sink, window, sel_bits, scale, out, ws, st,
                                             part_out, nullptr);
    }
    return sparse ? launch_t<64, true>(d, Q, K, V, ctx_len, sink, window, sel_bits, scale, out, ws, st, part_out,
                                       plan)
                  : launch_t<64, false>(d, Q, K, V, ctx_len, sink, window, sel_bits, scale, out, ws, st, part_out,
                                        nullptr);
}

cudaError_t launch_attn_plan(const tb_dims &d, const uint32_t *sel_bits, const int32_t *ctx_len, int32_t sink,
                             int32_t window, int32_t *plan, uint32_t *flags, cudaStream_t st) {
    const int W = (d.ctx_cap + 31) / 32;
    return launch_pdl(attn_plan_kernel, dim3(d.n_kv_heads, d.batch), dim3(kPlanThreads), 0, st, sel_bits, ctx_len,
                      d.n_q_heads, d.n_kv_heads, d.ctx_cap, W, sink, window, attn_splits(d), plan, flags);
}

cudaError_t launch_combine(const float *parts, int32_t n_parts, int32_t rows, int32_t head_dim, float *out,
                           cudaStream_t st) {
    if (head_dim == 128)
        return launch_pdl(combine_kernel<128>, dim3(rows), dim3(128), 0, st, parts, n_parts, rows, out);
    return launch_pdl(combine_kernel<64>, dim3(rows), dim3(64), 0, st, parts, n_parts, rows, out);
}

}  // namespace tb
