// Importance scores q'.k' of K' rows, shared by the selection kernels so that
// every selection path ranks bit-identical fp32 scores.
//
// TokenButler technical summary (gist.science), "Core architecture: scoring":
// a token's importance for a head is the dot product of the head's predicted
// query q' (d' fp32) with the token's projected key k' (d' bf16).  A KV
// group's 4 query heads share the key, so each row is read once for 4 heads.
//
// A warp works on blocks of 32 consecutive rows, staged in a shared-memory
// slot of its own by 16-byte cp.async copies: in copy i, lane l fetches part
// l % NPART of row i * (32 / NPART) + l / NPART (NPART = d' / 8 parts of 16
// bytes per row), so each copy instruction reads one contiguous 512-byte span
// of K'.  A row's parts land rotated by a few 16-byte slots (by (row >> 1) & 3
// for d' = 32, (row >> 2) & 1 for d' = 16), so that afterwards lane l can read
// all of row l with 16-byte loads that hit distinct banks.  Lane l then scores
// row l for the 4 heads with paired fp32 FMAs, the queries read from shared
// memory (the same address for every lane).  The summation order of a score
// is fixed:
//   score = (e0 + e2 + e4 + ... in order) + (e1 + e3 + e5 + ... in order)
// two FMA chains (even and odd elements of q' * k', each starting from 0)
// added at the end, so the rounding error stays within d'/2 + 1 roundings of
// sum |q_i k_i|.
#pragma once

#include "common.cuh"

namespace tb {

__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
// The two bf16 of a packed word as an fp32 pair (element 0 in the low half).
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t w) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(w << 16), "r"(w & 0xffff0000u));
    return r;
}
// Element-wise a * b + c on fp32 pairs, each rounded to nearest even.
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ float sum_f32x2(uint64_t v) {
    float a, b;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
    return a + b;
}

template <int DP>
struct BlockScorer {
    static_assert(DP == 16 || DP == 32, "d' of 16 or 32");
    static constexpr int NPART = DP / 8;  // 16-byte parts per row
    static constexpr int ROWB = DP * 2;    // bytes per row
    static constexpr int BLKB = 32 * ROWB; // bytes per 32-row block

    __device__ __forceinline__ static int rot(int row) {
        return NPART == 4 ? (row >> 1) & 3 : (row >> 2) & 1;
    }

    // Stage the block whose first row is `rows` (global, row r at rows + r *
    // DP) into the slot at shared address `slot`; rows r >= n_valid are not
    // read (zero-filled).  Whole warp; the caller commits and waits for the
    // copies (cp.async groups) and syncs the warp before score().
    __device__ __forceinline__ static void copy(uint32_t slot, const uint16_t *rows, int n_valid, int lane) {
#pragma unroll
        for (int i = 0; i < NPART; ++i) {
            const int c = i * 32 + lane;
            const int row = c / NPART, part = c % NPART;
            cp_async16(slot + row * ROWB + ((part + rot(row)) % NPART) * 16, rows + (size_t)row * DP + part * 8,
                       row < n_valid);
        }
    }

    // The scores of row `lane` of the staged block for the 4 heads (qs:
    // [4][DP] fp32 in shared memory).
    __device__ __forceinline__ static void score(const uint8_t *slot, const float *qs, int lane, float s[4]) {
        const uint8_t *row = slot + lane * ROWB;
        const int rt = rot(lane);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int v = 0; v < NPART; ++v) {  // the row's words 4v .. 4v+3, in order
            const uint4 raw = *reinterpret_cast<const uint4 *>(row + ((v + rt) % NPART) * 16);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float4 qa = *reinterpret_cast<const float4 *>(qs + h * DP + 8 * v);
                const float4 qb = *reinterpret_cast<const float4 *>(qs + h * DP + 8 * v + 4);
                acc[h] = fma_f32x2(pack_f32x2(qa.x, qa.y), bf16x2_to_f32x2(raw.x), acc[h]);
                acc[h] = fma_f32x2(pack_f32x2(qa.z, qa.w), bf16x2_to_f32x2(raw.y), acc[h]);
                acc[h] = fma_f32x2(pack_f32x2(qb.x, qb.y), bf16x2_to_f32x2(raw.z), acc[h]);
                acc[h] = fma_f32x2(pack_f32x2(qb.z, qb.w), bf16x2_to_f32x2(raw.w), acc[h]);
            }
        }
#pragma unroll
        for (int h = 0; h < 4; ++h) s[h] = sum_f32x2(acc[h]);
    }

    // score() for row `lane` of two staged blocks at once: every query load
    // serves both rows (the operations on each row are those of score()).
    __device__ __forceinline__ static void score2(const uint8_t *slot_a, const uint8_t *slot_b, const float *qs,
                                                  int lane, float sa[4], float sb[4]) {
        const uint8_t *row_a = slot_a + lane * ROWB;
        const uint8_t *row_b = slot_b + lane * ROWB;
        const int rt = rot(lane);
        uint64_t acc_a[4] = {0ull, 0ull, 0ull, 0ull}, acc_b[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int v = 0; v < NPART; ++v) {
            const uint4 ra = *reinterpret_cast<const uint4 *>(row_a + ((v + rt) % NPART) * 16);
            const uint4 rb = *reinterpret_cast<const uint4 *>(row_b + ((v + rt) % NPART) * 16);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float4 qa = *reinterpret_cast<const float4 *>(qs + h * DP + 8 * v);
                const float4 qb = *reinterpret_cast<const float4 *>(qs + h * DP + 8 * v + 4);
                const uint64_t q0 = pack_f32x2(qa.x, qa.y), q1 = pack_f32x2(qa.z, qa.w);
                const uint64_t q2 = pack_f32x2(qb.x, qb.y), q3 = pack_f32x2(qb.z, qb.w);
                acc_a[h] = fma_f32x2(q0, bf16x2_to_f32x2(ra.x), acc_a[h]);
                acc_a[h] = fma_f32x2(q1, bf16x2_to_f32x2(ra.y), acc_a[h]);
                acc_a[h] = fma_f32x2(q2, bf16x2_to_f32x2(ra.z), acc_a[h]);
                acc_a[h] = fma_f32x2(q3, bf16x2_to_f32x2(ra.w), acc_a[h]);
                acc_b[h] = fma_f32x2(q0, bf16x2_to_f32x2(rb.x), acc_b[h]);
                acc_b[h] = fma_f32x2(q1, bf16x2_to_f32x2(rb.y), acc_b[h]);
                acc_b[h] = fma_f32x2(q2, bf16x2_to_f32x2(rb.z), acc_b[h]);
                acc_b[h] = fma_f32x2(q3, bf16x2_to_f32x2(rb.w), acc_b[h]);
            }
        }
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            sa[h] = sum_f32x2(acc_a[h]);
            sb[h] = sum_f32x2(acc_b[h]);
        }
    }
};

}  // namespace tb
