// Importance scores q'.k' of staged K' rows, shared by the selection kernels
// so that every selection path ranks bit-identical fp32 scores.
//
// TokenButler technical summary (gist.science), "Core architecture: scoring":
// a token's importance for a head is the dot product of the head's predicted
// query q' (d' fp32) with the token's projected key k' (d' bf16).  A KV
// group's 4 query heads share the key, so each row is read once for 4 heads.
//
// A warp scores 32 consecutive rows staged in shared memory.  A row of DP
// bf16 is NPART = DP / 8 parts of 16 bytes; in pass i lane l reads part
// l % NPART of row i * (32 / NPART) + l / NPART, so a warp's 16-byte reads
// are consecutive and free of bank conflicts.  The lane forms its part's
// partial dot product for the 4 heads with paired fp32 FMAs (even and odd
// elements in separate chains, then added), and a butterfly over the row's
// NPART lanes leaves each lane the full score of 4 / NPART heads.  The
// summation order of a score is fixed whatever lane computes it:
//   part  = (e0 e2 e4 e6 chain) + (e1 e3 e5 e7 chain)
//   score = (part0 + part2) + (part1 + part3)   for d' = 32
//   score = part0 + part1                       for d' = 16
// so the rounding error stays within 7 roundings of sum |q_i k_i|.
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
struct RowScorer {
    static_assert(DP == 16 || DP == 32, "d' of 16 or 32");
    static constexpr int NPART = DP / 8;   // 16-byte parts per row
    static constexpr int RPP = 32 / NPART;  // rows per pass
    static constexpr int HPL = 4 / NPART;   // heads a lane holds after a pass
    static constexpr int ROWB = DP * 2;     // bytes per row
    uint64_t q2[4][4];                      // this lane's part of the 4 queries, as fp32 pairs

    // qs: [4][DP] fp32 in shared memory.
    __device__ __forceinline__ void load_q(const float *qs, int lane) {
        const int part = lane % NPART;
#pragma unroll
        for (int h = 0; h < 4; ++h)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 v = *reinterpret_cast<const float2 *>(qs + h * DP + part * 8 + 2 * i);
                q2[h][i] = pack_f32x2(v.x, v.y);
            }
    }
    // The first head whose score lane `lane` holds after a pass (then +1 .. HPL-1).
    __device__ __forceinline__ static int head0(int lane) { return (lane % NPART) * HPL; }
    // The row (within the 32-row block) lane `lane` holds after pass `pass`.
    __device__ __forceinline__ static int row_of(int pass, int lane) { return pass * RPP + lane / NPART; }
    // Shared-memory address of the part lane `lane` reads in pass `pass` of
    // the block at `block` (32 rows of ROWB bytes).
    __device__ __forceinline__ static const uint4 *part_ptr(const uint8_t *block, int pass, int lane) {
        return reinterpret_cast<const uint4 *>(block + (pass * 32 + lane) * 16);
    }

    // One pass over `raw`, the 16-byte part this lane read: out[j] = score of
    // head head0(lane) + j for row row_of(pass, lane).  Whole warp.
    __device__ __forceinline__ void pass(const uint4 raw, int lane, float out[HPL]) const {
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint64_t k = bf16x2_to_f32x2(w[i]);
#pragma unroll
            for (int h = 0; h < 4; ++h) acc[h] = fma_f32x2(q2[h][i], k, acc[h]);
        }
        finish(acc, lane, out);
    }
    // The same pass with the queries read from shared memory (qs: [4][DP]
    // fp32) instead of registers: the same operations in the same order, so
    // the same scores, for kernels that need the registers for other things.
    __device__ __forceinline__ static void pass_q(const float *qs, const uint4 raw, int lane, float out[HPL]) {
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        const int part = lane % NPART;
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const float4 lo = *reinterpret_cast<const float4 *>(qs + h * DP + part * 8);
            const float4 hi = *reinterpret_cast<const float4 *>(qs + h * DP + part * 8 + 4);
            acc[h] = fma_f32x2(pack_f32x2(lo.x, lo.y), bf16x2_to_f32x2(w[0]), acc[h]);
            acc[h] = fma_f32x2(pack_f32x2(lo.z, lo.w), bf16x2_to_f32x2(w[1]), acc[h]);
            acc[h] = fma_f32x2(pack_f32x2(hi.x, hi.y), bf16x2_to_f32x2(w[2]), acc[h]);
            acc[h] = fma_f32x2(pack_f32x2(hi.z, hi.w), bf16x2_to_f32x2(w[3]), acc[h]);
        }
        finish(acc, lane, out);
    }

  private:
    // Each head's even and odd chains added, then the butterfly over the row's lanes.
    __device__ __forceinline__ static void finish(const uint64_t acc[4], int lane, float out[HPL]) {
        float s[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) s[h] = sum_f32x2(acc[h]);
        const int p = lane % NPART;
        if constexpr (NPART == 4) {
            // lanes p and p^2 trade the heads the other keeps, then p and p^1
            const bool up = (p & 2) != 0;
            const float u0 = (up ? s[2] : s[0]) + __shfl_xor_sync(0xffffffffu, up ? s[0] : s[2], 2);
            const float u1 = (up ? s[3] : s[1]) + __shfl_xor_sync(0xffffffffu, up ? s[1] : s[3], 2);
            const bool odd = (p & 1) != 0;
            out[0] = (odd ? u1 : u0) + __shfl_xor_sync(0xffffffffu, odd ? u0 : u1, 1);
        } else {
            const bool odd = (p & 1) != 0;
            out[0] = (odd ? s[2] : s[0]) + __shfl_xor_sync(0xffffffffu, odd ? s[0] : s[2], 1);
            out[1] = (odd ? s[3] : s[1]) + __shfl_xor_sync(0xffffffffu, odd ? s[1] : s[3], 1);
        }
    }

  public:
    // The 4 head scores of the lane's row brought to the row's first lane
    // (part 0), heads in order.  Whole warp; valid at lanes with part 0.
    __device__ __forceinline__ static void gather_heads(const float out[HPL], float s[4]) {
        if constexpr (NPART == 4) {
            s[0] = out[0];
            s[1] = __shfl_down_sync(0xffffffffu, out[0], 1);
            s[2] = __shfl_down_sync(0xffffffffu, out[0], 2);
            s[3] = __shfl_down_sync(0xffffffffu, out[0], 3);
        } else {
            s[0] = out[0];
            s[1] = out[1];
            s[2] = __shfl_down_sync(0xffffffffu, out[0], 1);
            s[3] = __shfl_down_sync(0xffffffffu, out[1], 1);
        }
    }
};

}  // namespace tb
