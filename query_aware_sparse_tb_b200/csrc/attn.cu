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
// Work split: one CTA per (sequence b, KV head g, context chunk).  The CTA
// builds the chunk's row list (sparse: union over the 4 query heads of the
// group of their selected bits, plus sink and window rows, each row tagged
// with a 4-bit head mask), then streams the K and V rows of that list through
// a 3-stage cp.async pipeline in shared memory, so every (b, g, t) row crosses
// HBM once for the whole group.  Each warp takes 8 rows of a 64-row tile; a
// half-warp owns 4 rows and each lane 1/16 of head_dim, so every K/V element
// a lane loads is used by all 4 query heads.  Partial dot products are summed
// across the 16 lanes of a row by a transposing butterfly (15 shuffles for 16
// sums), the online-softmax state is per warp, and the last CTA of each
// (b, g) — found with an atomic ticket, never a wait — merges the chunks'
// partial states into the fp32 output.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace tb {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTile = 64;       // rows per pipeline stage
constexpr int kStages = 3;
constexpr int kGroup = 4;       // query heads per KV head
constexpr int kMaxChunk = 2048; // positions per row list (a CTA walks its range in sub-chunks)
constexpr int kMaxSplits = 64;   // partial states merged per (sequence, KV head)
constexpr unsigned kFull = 0xffffffffu;

template <int D>
struct Smem {
    static constexpr int kStageBytes = 2 * kTile * D * 2;  // K tile + V tile, bf16
    static constexpr int kPipe = kStages * kStageBytes;
    static constexpr int kList = kMaxChunk * 4;
    static constexpr int kP = kWarps * 32 * 4;
    static constexpr int kWords = (kMaxChunk / 32) * 4;
    // per-warp transpose buffer (16 values x 32 lanes): at D = 128 it overlays
    // the warp's own 8 K rows of the current stage (2 KB), at D = 64 it has its
    // own space
    static constexpr int kRed = D == 128 ? 0 : kWarps * 16 * 32 * 4;
    static constexpr int kTotal = kPipe + kList + kP + kWords + kRed;
    // the pipeline region is reused for the end-of-CTA combine and the merge
    static_assert(kWarps * kGroup * (D + 2) * 4 <= kPipe, "combine scratch");
    static_assert(kMaxSplits * kGroup * 4 <= kPipe, "merge scratch");
};

__device__ __forceinline__ float pick4(const float (&v)[4], int i) {
    return i == 0 ? v[0] : i == 1 ? v[1] : i == 2 ? v[2] : v[3];
}
__device__ __forceinline__ float comp4(const float4 &v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Raw DPL bf16 values of one row chunk (8 -> uint4, 4 -> uint2 in .x/.y).
template <int DPL>
__device__ __forceinline__ uint4 load_raw(const uint16_t *p) {
    if constexpr (DPL == 8) {
        return *reinterpret_cast<const uint4 *>(p);
    } else {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        return make_uint4(u.x, u.y, 0u, 0u);
    }
}
// bf16 pairs -> fp32 pairs (element 2e in .x, 2e+1 in .y).
template <int DPL>
__device__ __forceinline__ void unpack2(const uint4 &u, float2 (&f)[DPL / 2]) {
    f[0] = make_float2(bf16_lo(u.x), bf16_hi(u.x));
    f[1] = make_float2(bf16_lo(u.y), bf16_hi(u.y));
    if constexpr (DPL == 8) {
        f[2] = make_float2(bf16_lo(u.z), bf16_hi(u.z));
        f[3] = make_float2(bf16_lo(u.w), bf16_hi(u.w));
    }
}

template <int D, bool SPARSE>
__global__ void __launch_bounds__(kThreads, 2)
attn_kernel(const uint16_t *__restrict__ Q, const uint16_t *__restrict__ K,
            const uint16_t *__restrict__ V, const int32_t *__restrict__ ctx_len,
            const uint32_t *__restrict__ sel_bits, int Hq, int Hkv, int Tcap, int W, int sink,
            int window, float qscale, int splits, float *__restrict__ part,
            uint32_t *__restrict__ counters, float *__restrict__ out, uint32_t *__restrict__ flags) {
    constexpr int DPL = D / 16;  // head_dim elements per lane
    constexpr int CPR = D / 8;   // 16-byte chunks per row
    constexpr int kCopies = kTile * CPR / kThreads;
    // one partial state per head: O[D], M, L, 2 pad floats, so every head's
    // record starts 16-byte aligned for the float4 loads of the merge
    constexpr int kHS = D + 4;
    constexpr int kPartStride = kGroup * kHS;
    using S = Smem<D>;

    extern __shared__ __align__(1024) uint8_t smem[];
    uint16_t *pipe = reinterpret_cast<uint16_t *>(smem);
    int32_t *list = reinterpret_cast<int32_t *>(smem + S::kPipe);
    float *pbuf = reinterpret_cast<float *>(smem + S::kPipe + S::kList);
    int32_t *wcnt = reinterpret_cast<int32_t *>(smem + S::kPipe + S::kList + S::kP);
    __shared__ int s_nrows, s_last;
    __shared__ float s_red[kWarps][kGroup];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int half = lane >> 4, c = lane & 15;
    const int b = blockIdx.z, g = blockIdx.y, split = blockIdx.x;
    const int T = clamp_ctx(ctx_len[b], Tcap, flags, tid == 0 && split == 0 && g == 0);
    // this sequence's length split evenly over the CTAs of (b, g), in 64-row units
    const int chunk = ((T + splits - 1) / splits + kTile - 1) / kTile * kTile;
    const int ns = (T + chunk - 1) / chunk;  // CTAs of (b, g) that hold rows
    const int p_begin = split * chunk;
    const int p_end = min(p_begin + chunk, T);
    const size_t slab = ((size_t)b * Hkv + g) * (size_t)Tcap;
    const uint16_t *Kb = K + slab * D;
    const uint16_t *Vb = V + slab * D;
    float *part_bg = part + (size_t)(b * Hkv + g) * splits * kPartStride;

    if (p_begin < T) {
        // ------------------------------------------------ per-lane query slice
        // (pairs of dims, pre-scaled into log2 units)
        constexpr int DP2 = DPL / 2;
        float2 q2[kGroup][DP2];
#pragma unroll
        for (int h = 0; h < kGroup; ++h) {
            const uint16_t *qp = Q + ((size_t)b * Hq + g * kGroup + h) * D + c * DPL;
            uint4 u;
            if constexpr (DPL == 8) {
                u = __ldg(reinterpret_cast<const uint4 *>(qp));
            } else {
                const uint2 v = __ldg(reinterpret_cast<const uint2 *>(qp));
                u = make_uint4(v.x, v.y, 0u, 0u);
            }
            unpack2<DPL>(u, q2[h]);
#pragma unroll
            for (int e = 0; e < DP2; ++e) q2[h][e] = __fmul2_rn(q2[h][e], make_float2(qscale, qscale));
        }

        // online-softmax state: m_run is a shared reference per head, raised
        // only when a logit exceeds it by more than kLazy (log2 units), so every
        // weight exp2(x - m_run) stays <= 2^kLazy; the result is the same
        // softmax, m_run just need not be the running maximum
        constexpr float kLazy = 8.0f;
        float m_run[kGroup];
        float2 l2[2];
        float2 acc2[kGroup][DP2];
#pragma unroll
        for (int h = 0; h < kGroup; ++h) {
            m_run[h] = -INFINITY;
#pragma unroll
            for (int e = 0; e < DP2; ++e) acc2[h][e] = make_float2(0.f, 0.f);
        }
        l2[0] = l2[1] = make_float2(0.f, 0.f);
        const uint32_t pipe_s = smem_addr(pipe);
        const int rb = warp * 8 + half * 4;  // this half-warp's first row in a tile

        // the CTA's range in sub-chunks of at most kMaxChunk positions
        for (int p0 = p_begin; p0 < p_end; p0 += kMaxChunk) {
            const int p1 = min(p0 + kMaxChunk, p_end);
            // -------------------------------------------- row list (sparse)
            int n_rows = p1 - p0;
            if constexpr (SPARSE) {
                const int hi_c = T - window;  // candidates are [sink, hi_c)
                const int nwords = (p1 - p0 + 31) >> 5;
                const int w0 = p0 >> 5;
                const uint32_t *sb = sel_bits + ((size_t)b * Hq + (size_t)g * kGroup) * W + w0;
                auto word_mask = [&](int wi, int &p, int &m) -> uint32_t {
                    uint32_t hb = lane < kGroup ? __ldg(sb + (size_t)lane * W + wi) : 0u;
                    uint32_t b0 = __shfl_sync(kFull, hb, 0), b1 = __shfl_sync(kFull, hb, 1);
                    uint32_t b2 = __shfl_sync(kFull, hb, 2), b3 = __shfl_sync(kFull, hb, 3);
                    p = p0 + (wi << 5) + lane;
                    m = 0;
                    if (p < p1) {
                        if (p < sink || p >= hi_c) {
                            m = 0xF;
                        } else {
                            m = ((b0 >> lane) & 1u) | (((b1 >> lane) & 1u) << 1) |
                                (((b2 >> lane) & 1u) << 2) | (((b3 >> lane) & 1u) << 3);
                        }
                    }
                    return __ballot_sync(kFull, m != 0);
                };
                for (int wi = warp; wi < nwords; wi += kWarps) {
                    int p, m;
                    uint32_t bal = word_mask(wi, p, m);
                    if (lane == 0) wcnt[wi] = __popc(bal);
                }
                __syncthreads();
                if (warp == 0) {  // exclusive scan of <= 64 word counts
                    int a0 = (2 * lane < nwords) ? wcnt[2 * lane] : 0;
                    int a1 = (2 * lane + 1 < nwords) ? wcnt[2 * lane + 1] : 0;
                    int sum = a0 + a1, incl = sum;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        int v = __shfl_up_sync(kFull, incl, o);
                        if (lane >= o) incl += v;
                    }
                    int excl = incl - sum;
                    if (2 * lane < nwords) wcnt[2 * lane] = excl;
                    if (2 * lane + 1 < nwords) wcnt[2 * lane + 1] = excl + a0;
                    if (lane == 31) s_nrows = incl;
                }
                __syncthreads();
                for (int wi = warp; wi < nwords; wi += kWarps) {
                    int p, m;
                    uint32_t bal = word_mask(wi, p, m);
                    if (m) list[wcnt[wi] + __popc(bal & ((1u << lane) - 1u))] = (p << 4) | m;
                }
                __syncthreads();
                n_rows = s_nrows;
            }

            const int n_tiles = (n_rows + kTile - 1) / kTile;
            auto issue = [&](int t) {
                const uint32_t kbase = pipe_s + (t % kStages) * S::kStageBytes;
                const uint32_t vbase = kbase + kTile * D * 2;
#pragma unroll
                for (int k = 0; k < kCopies; ++k) {
                    const int e = tid + k * kThreads;
                    const int r = e / CPR, ch = e % CPR;
                    const int gr = t * kTile + r;
                    const bool valid = gr < n_rows;
                    int pos = p0;
                    if (valid) pos = SPARSE ? (list[gr] >> 4) : (p0 + gr);
                    const size_t off = (size_t)pos * D + ch * 8;
                    const uint32_t so = (uint32_t)(r * D + ch * 8) * 2u;
                    cp_async16(kbase + so, Kb + off, valid);
                    cp_async16(vbase + so, Vb + off, valid);
                }
            };

#pragma unroll
            for (int s = 0; s < kStages - 1; ++s) {
                if (s < n_tiles) issue(s);
                cp_async_commit();
            }

            for (int t = 0; t < n_tiles; ++t) {
                cp_async_wait<kStages - 2>();
                __syncthreads();
                if (t + kStages - 1 < n_tiles) issue(t + kStages - 1);
                cp_async_commit();

                const uint16_t *Ks = pipe + (t % kStages) * (S::kStageBytes / 2);
                const uint16_t *Vs = Ks + kTile * D;

                // partial q.k over this lane's slice: 4 rows x 4 heads
                uint4 kr[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) kr[j] = load_raw<DPL>(Ks + (rb + j) * D + c * DPL);
                float s[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float2 k2[DP2];
                    unpack2<DPL>(kr[j], k2);
#pragma unroll
                    for (int h = 0; h < kGroup; ++h) {
                        float2 a = __fmul2_rn(q2[h][0], k2[0]);
#pragma unroll
                        for (int e = 1; e < DP2; ++e) a = __ffma2_rn(q2[h][e], k2[e], a);
                        s[j * 4 + h] = a.x + a.y;
                    }
                }
                // transpose through shared memory: value v = (row v>>2, head
                // v&3) of lane l goes to red[v][l ^ swz(v)]; lane c of each
                // half then sums the 16 values (row c>>2, head c&3) of its
                // half.  The XOR swizzle keeps both sides bank-conflict free.
                float *red;
                if constexpr (D == 128) {
                    red = reinterpret_cast<float *>(const_cast<uint16_t *>(Ks) + warp * 8 * D);
                } else {
                    red = reinterpret_cast<float *>(smem + S::kPipe + S::kList + S::kP + S::kWords) +
                          warp * 16 * 32;
                }
                __syncwarp();  // every lane holds its K chunks before the rows are overwritten
#pragma unroll
                for (int v = 0; v < 16; ++v) red[v * 32 + (lane ^ ((v & 7) << 2))] = s[v];
                __syncwarp();
                float x;
                {
                    const float *rp = red + c * 32;
                    const int sw = (c & 7) << 2;
                    const float4 r0 = *reinterpret_cast<const float4 *>(rp + ((half * 16 + 0) ^ sw));
                    const float4 r1 = *reinterpret_cast<const float4 *>(rp + ((half * 16 + 4) ^ sw));
                    const float4 r2 = *reinterpret_cast<const float4 *>(rp + ((half * 16 + 8) ^ sw));
                    const float4 r3 = *reinterpret_cast<const float4 *>(rp + ((half * 16 + 12) ^ sw));
                    float2 a0 = __fadd2_rn(make_float2(r0.x, r0.y), make_float2(r0.z, r0.w));
                    float2 a1 = __fadd2_rn(make_float2(r1.x, r1.y), make_float2(r1.z, r1.w));
                    float2 a2 = __fadd2_rn(make_float2(r2.x, r2.y), make_float2(r2.z, r2.w));
                    float2 a3 = __fadd2_rn(make_float2(r3.x, r3.y), make_float2(r3.z, r3.w));
                    a0 = __fadd2_rn(__fadd2_rn(a0, a1), __fadd2_rn(a2, a3));
                    x = a0.x + a0.y;
                }
                const int hh = c & 3;
                {
                    const int gr = t * kTile + rb + (c >> 2);
                    uint32_t mk = 0;
                    if (gr < n_rows) mk = SPARSE ? (uint32_t)(list[gr] & 0xF) : 0xFu;
                    if (!((mk >> hh) & 1u)) x = -INFINITY;
                }
                // raise the per-head references only when some logit of the
                // warp's 8 rows exceeds its reference by more than kLazy
                if (__any_sync(kFull, x > pick4(m_run, hh) + kLazy)) {
                    float mx = x;
                    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
#pragma unroll
                    for (int h = 0; h < kGroup; ++h) {
                        const float mn = fmaxf(m_run[h], __shfl_sync(kFull, mx, h));
                        if (mn > m_run[h]) {
                            const float alpha = exp2f(m_run[h] - mn);  // 0 while m_run is -inf
                            const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
                            for (int e = 0; e < DP2; ++e) acc2[h][e] = __fmul2_rn(acc2[h][e], a2);
                            if (h == 0) l2[0].x *= alpha;
                            if (h == 1) l2[0].y *= alpha;
                            if (h == 2) l2[1].x *= alpha;
                            if (h == 3) l2[1].y *= alpha;
                            m_run[h] = mn;
                        }
                    }
                }
                const float p = (x == -INFINITY) ? 0.f : exp2f(x - pick4(m_run, hh));
                __syncwarp();  // transpose values read before the slot is reused
                red[lane] = p;
                __syncwarp();
                float4 pr[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) pr[j] = *reinterpret_cast<const float4 *>(red + half * 16 + j * 4);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    l2[0] = __fadd2_rn(l2[0], make_float2(pr[j].x, pr[j].y));
                    l2[1] = __fadd2_rn(l2[1], make_float2(pr[j].z, pr[j].w));
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float2 v2[DP2];
                    unpack2<DPL>(load_raw<DPL>(Vs + (rb + j) * D + c * DPL), v2);
#pragma unroll
                    for (int h = 0; h < kGroup; ++h) {
                        const float ph = comp4(pr[j], h);
                        const float2 pp = make_float2(ph, ph);
#pragma unroll
                        for (int e = 0; e < DP2; ++e) acc2[h][e] = __ffma2_rn(pp, v2[e], acc2[h][e]);
                    }
                }
            }
            cp_async_wait<0>();
            __syncthreads();  // pipeline and list free for the next sub-chunk
        }

        // ------------------------------------------------ combine halves, warps
        float l[kGroup] = {l2[0].x, l2[0].y, l2[1].x, l2[1].y};
        float acc[kGroup][DPL];
#pragma unroll
        for (int h = 0; h < kGroup; ++h) {
            l[h] += __shfl_xor_sync(kFull, l[h], 16);
#pragma unroll
            for (int e = 0; e < DP2; ++e) {
                acc[h][2 * e] = acc2[h][e].x + __shfl_xor_sync(kFull, acc2[h][e].x, 16);
                acc[h][2 * e + 1] = acc2[h][e].y + __shfl_xor_sync(kFull, acc2[h][e].y, 16);
            }
        }
        float *cacc = reinterpret_cast<float *>(smem);           // [warp][head][D]
        float *cml = cacc + kWarps * kGroup * D;                 // [warp][head][m, l]
        if (half == 0) {
#pragma unroll
            for (int h = 0; h < kGroup; ++h)
#pragma unroll
                for (int e = 0; e < DPL; ++e) cacc[(warp * kGroup + h) * D + c * DPL + e] = acc[h][e];
        }
        if (lane == 0) {
#pragma unroll
            for (int h = 0; h < kGroup; ++h) {
                cml[(warp * kGroup + h) * 2] = m_run[h];
                cml[(warp * kGroup + h) * 2 + 1] = l[h];
            }
        }
        __syncthreads();
        float *pp = part_bg + (size_t)split * kPartStride;
        for (int it = tid; it < kGroup * D; it += kThreads) {
            const int h = it / D, dim = it % D;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) M = fmaxf(M, cml[(w * kGroup + h) * 2]);
            float O = 0.f, L = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kWarps; ++w) {
                    const float mw = cml[(w * kGroup + h) * 2];
                    if (mw != -INFINITY) {
                        const float f = exp2f(mw - M);
                        O = fmaf(cacc[(w * kGroup + h) * D + dim], f, O);
                        L = fmaf(cml[(w * kGroup + h) * 2 + 1], f, L);
                    }
                }
            }
            pp[h * kHS + dim] = O;
            if (dim == 0) {
                pp[h * kHS + D] = M;
                pp[h * kHS + D + 1] = L;
            }
        }
    }

    // ---------------------------------------------------- last CTA merges
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned prev = atomicAdd(&counters[b * Hkv + g], 1u);
        s_last = (prev == (unsigned)splits - 1u);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // weights w[s][h] = exp2(M_sh - M*_h) / L*_h over the ns <= 64 partials:
    // one (split, head) pair per thread, head = tid & 3
    float *wsm = reinterpret_cast<float *>(smem);  // [ns][head]
    {
        const int h = tid & 3, s = tid >> 2;
        float m = -INFINITY, lw = 0.f;
        if (s < ns) {
            m = __ldcg(part_bg + (size_t)s * kPartStride + h * kHS + D);
            lw = __ldcg(part_bg + (size_t)s * kPartStride + h * kHS + D + 1);
        }
        float mx = m;
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
        if (lane < kGroup) s_red[warp][lane] = mx;
        __syncthreads();
        float Mh = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) Mh = fmaxf(Mh, s_red[w][h]);
        const float f = (m == -INFINITY) ? 0.f : exp2f(m - Mh);
        float lsum = f * lw;
        lsum += __shfl_xor_sync(kFull, lsum, 4);
        lsum += __shfl_xor_sync(kFull, lsum, 8);
        lsum += __shfl_xor_sync(kFull, lsum, 16);
        __syncthreads();
        if (lane < kGroup) s_red[warp][lane] = lsum;
        __syncthreads();
        float Lh = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) Lh += s_red[w][h];
        if (s < ns) wsm[s * kGroup + h] = Lh > 0.f ? f / Lh : 0.f;
    }
    __syncthreads();
    // outputs as float4 groups (head, 4 dims); TPG threads per group split the
    // partials and combine with shuffles; loads are issued 8 at a time
    constexpr int kGroups4 = kGroup * D / 4;
    constexpr int TPG = kThreads / kGroups4;
    {
        const int grp = tid / TPG, j = tid % TPG;
        const int h = grp / (D / 4), d4 = grp % (D / 4);
        const float *src = part_bg + h * kHS + d4 * 4;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s0 = j; s0 < ns; s0 += 8 * TPG) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int s = s0 + u * TPG;
                v[u] = s < ns ? __ldcg(reinterpret_cast<const float4 *>(src + (size_t)s * kPartStride))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int s = s0 + u * TPG;
                const float wgt = s < ns ? wsm[s * kGroup + h] : 0.f;
                o.x = fmaf(v[u].x, wgt, o.x); o.y = fmaf(v[u].y, wgt, o.y);
                o.z = fmaf(v[u].z, wgt, o.z); o.w = fmaf(v[u].w, wgt, o.w);
            }
        }
#pragma unroll
        for (int off = 1; off < TPG; off <<= 1) {
            o.x += __shfl_xor_sync(kFull, o.x, off); o.y += __shfl_xor_sync(kFull, o.y, off);
            o.z += __shfl_xor_sync(kFull, o.z, off); o.w += __shfl_xor_sync(kFull, o.w, off);
        }
        if (j == 0) {  // scalar stores: `out` is only required to be 4-byte aligned
            float *dst = out + ((size_t)b * Hq + g * kGroup + h) * D + d4 * 4;
            dst[0] = o.x; dst[1] = o.y; dst[2] = o.z; dst[3] = o.w;
        }
    }
    if (tid == 0) counters[b * Hkv + g] = 0u;  // leave the ticket zeroed for the next call
}

int g_num_sms = 0;

int num_sms() {
    if (g_num_sms == 0) {
        int dev = 0, n = 148;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
            g_num_sms = n;
        else
            g_num_sms = 148;
    }
    return g_num_sms;
}

template <int D, bool SPARSE>
cudaError_t launch_t(const tb_dims &d, const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                     const int32_t *ctx_len, int32_t sink, int32_t window, const uint32_t *sel_bits,
                     float scale, float *out, void *ws, cudaStream_t st) {
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(attn_kernel<D, SPARSE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             Smem<D>::kTotal);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const int splits = attn_splits(d);
    uint8_t *w = static_cast<uint8_t *>(ws);
    uint32_t *flags = reinterpret_cast<uint32_t *>(w);
    uint32_t *counters = reinterpret_cast<uint32_t *>(w + kWsHeaderBytes);
    float *part = reinterpret_cast<float *>(
        w + kWsHeaderBytes + align_up((size_t)d.batch * d.n_kv_heads * 4, 256));
    const int W = (d.ctx_cap + 31) / 32;
    const float qscale = scale * 1.4426950408889634f;  // logits in log2 units for exp2
    dim3 grid(splits, d.n_kv_heads, d.batch);
    attn_kernel<D, SPARSE><<<grid, kThreads, Smem<D>::kTotal, st>>>(
        Q, K, V, ctx_len, sel_bits, d.n_q_heads, d.n_kv_heads, d.ctx_cap, W, sink, window, qscale,
        splits, part, counters, out, flags);
    return cudaGetLastError();
}

}  // namespace

// CTAs per (sequence, KV head): enough for one wave of two CTAs per SM over
// all (sequence, KV head) pairs, at most kMaxSplits, each with at least one
// 64-row tile of the longest sequence; among the candidates up to twice that,
// the count with the best wave quantisation.
int attn_splits(const tb_dims &d) {
    const long long slots = 2LL * num_sms();
    const long long pairs = (long long)d.batch * d.n_kv_heads;
    const int max_useful = (d.ctx_cap + kTile - 1) / kTile;
    int lo = (int)((slots + pairs - 1) / pairs);
    lo = std::max(1, std::min({lo, kMaxSplits, max_useful}));
    int best = lo;
    double best_eff = 0.0;
    for (int s = lo; s <= std::min({2 * lo, kMaxSplits, max_useful}); ++s) {
        const long long ctas = pairs * s;
        const double eff = (double)ctas / (double)(((ctas + slots - 1) / slots) * slots);
        if (eff > best_eff + 1e-9) {
            best_eff = eff;
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
                        cudaStream_t st) {
    if (d.head_dim == 128) {
        return sparse ? launch_t<128, true>(d, Q, K, V, ctx_len, sink, window, sel_bits, scale, out, ws, st)
                      : launch_t<128, false>(d, Q, K, V, ctx_len, sink, window, sel_bits, scale, out, ws, st);
    }
    return sparse ? launch_t<64, true>(d, Q, K, V, ctx_len, sink, window, sel_bits, scale, out, ws, st)
                  : launch_t<64, false>(d, Q, K, V, ctx_len, sink, window, sel_bits, scale, out, ws, st);
}

}  // namespace tb
