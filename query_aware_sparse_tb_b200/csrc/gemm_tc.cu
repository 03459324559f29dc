// Tensor-core (tcgen05) kernels: batched key projection and the query
// predictor MLP.
//
// TokenButler technical summary (gist.science), "Core architecture":
//   - key-cache projection: each consumer layer projects its real keys with a
//     learned matrix into the d' space (here K' = K W_k^T, one W_k per KV
//     head), run on batches of N new tokens ("Optimisations: batching");
//   - query prediction: a light MLP on the producer layer's hidden state emits
//     G slot-specific d'-dim queries per head (here two bias-free products with
//     SiLU between them, the activation rounded to bf16 in between).
//
// Both are real dense contractions, so they run on the 5th-generation tensor
// cores: operands are brought into shared memory by TMA in the 128-byte
// swizzled K-major layout, one elected thread issues tcgen05.mma into a TMEM
// accumulator, completion is signalled through tcgen05.commit on an mbarrier,
// and the epilogue reads TMEM with tcgen05.ld.  Every mbarrier wait is bounded
// (TB_FLAG_TIMEOUT on expiry) and TMEM is always released.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace tb {
namespace {

constexpr uint32_t kAtomA = 128 * 128;  // 128 rows x 128 B (64 bf16 of K)

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D bf16 tensor [outer][inner] (inner contiguous), box {64, box_outer},
// 128-byte swizzle, zero fill outside the tensor.
bool make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {64, box_outer};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------- key projection

// One CTA projects up to 128 rows of one (sequence, KV head):
// D[128 x d'] = A[128 x d] (keys, K-major) * B[d' x d]^T (W_k, K-major).
template <int D, int DP>
__global__ void __launch_bounds__(128)
project_keys_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmW,
                    uint16_t *__restrict__ Kp, const int32_t *__restrict__ tok_begin,
                    const int32_t *__restrict__ tok_count, int Hkv, int Tcap, uint32_t *flags) {
    constexpr int KA = D / 64;                 // swizzle atoms along K
    constexpr uint32_t kAtomB = DP * 128;      // DP rows x 128 B
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bars[2];
    __shared__ uint32_t tmem_slot;
    __shared__ int s_ok;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.z, g = blockIdx.y, tile = blockIdx.x;
    griddep_wait();
    griddep_launch_dependents();
    const int begin = tok_begin[b], cnt = tok_count[b];
    if (begin < 0 || cnt <= tile * 128) return;
    const int t0 = begin + tile * 128;
    if (t0 >= Tcap) return;
    const int rows = min(min(128, cnt - tile * 128), Tcap - t0);

    const uint32_t sbase = (smem_addr(smem_raw) + 1023u) & ~1023u;
    const uint32_t sA = sbase, sB = sbase + KA * kAtomA;
    const uint32_t bar_tma = smem_addr(&bars[0]), bar_mma = smem_addr(&bars[1]);

    if (warp == 0) {
        tmem_alloc(smem_addr(&tmem_slot), 32);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    if (tid == 0) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmW);
        mbar_arrive_expect_tx(bar_tma, KA * (kAtomA + kAtomB));
        const int y = (int)(((size_t)b * Hkv + g) * (size_t)Tcap + t0);
#pragma unroll
        for (int a = 0; a < KA; ++a) tma_load_2d(sA + a * kAtomA, &tmK, bar_tma, a * 64, y);
#pragma unroll
        for (int a = 0; a < KA; ++a) tma_load_2d(sB + a * kAtomB, &tmW, bar_tma, a * 64, g * DP);
        const bool ok = mbar_wait_bounded(bar_tma, 0, flags);
        if (ok) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_bf16_f32(128, DP);
#pragma unroll
            for (int kb = 0; kb < D / 16; ++kb) {
                const int a = kb >> 2, w = kb & 3;
                umma_bf16(tmem, sw128_kmajor_desc(sA + a * kAtomA + w * 32),
                          sw128_kmajor_desc(sB + a * kAtomB + w * 32), idesc, kb > 0 ? 1u : 0u);
            }
            umma_commit(bar_mma);
        }
        s_ok = ok ? 1 : 0;
    }
    __syncthreads();
    bool ok = s_ok != 0;
    if (ok) ok = mbar_wait_bounded(bar_mma, 0, flags);
    tc_fence_after();
    if (ok) {
        float r[DP];
        float (&r0)[16] = *reinterpret_cast<float (*)[16]>(&r[0]);
        tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16), r0);
        if constexpr (DP == 32) {
            float (&r1)[16] = *reinterpret_cast<float (*)[16]>(&r[16]);
            tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + 16, r1);
        }
        const int row = warp * 32 + lane;
        if (row < rows) {
            uint32_t packed[DP / 2];
#pragma unroll
            for (int j = 0; j < DP / 2; ++j)
                packed[j] = (uint32_t)f32_to_bf16_rne(r[2 * j]) | ((uint32_t)f32_to_bf16_rne(r[2 * j + 1]) << 16);
            uint4 *dst = reinterpret_cast<uint4 *>(Kp + (((size_t)b * Hkv + g) * (size_t)Tcap + t0 + row) * DP);
#pragma unroll
            for (int v = 0; v < DP / 8; ++v)
                dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 32);
}

// ------------------------------------------------------------ skinny GEMM

// partial[split][n][m] = sum over this split's K range of A[m][k] * B[n][k],
// A = weights [M][K] (K-major), B = activations [n_rows <= 16][K] (K-major,
// rows past n_rows read as zero by TMA).  One CTA: 128 rows of M, KB blocks of
// 64 along K, all loads in flight at once, one mbarrier per block so the MMAs
// start as soon as a block lands.
template <int KB>
__global__ void __launch_bounds__(128)
skinny_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   float *__restrict__ partial, int M, int n_rows, uint32_t *flags) {
    constexpr uint32_t kAtomB = 16 * 128;
    constexpr uint32_t kStage = kAtomA + kAtomB;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bars[KB + 1];
    __shared__ uint32_t tmem_slot;
    __shared__ int s_ok;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m0 = blockIdx.x * 128, split = blockIdx.y;
    const int k0 = split * KB * 64;
    const uint32_t sbase = (smem_addr(smem_raw) + 1023u) & ~1023u;

    if (warp == 0) {
        tmem_alloc(smem_addr(&tmem_slot), 32);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i <= KB; ++i) mbar_init(smem_addr(&bars[i]), 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    griddep_wait();
    griddep_launch_dependents();

    if (tid == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
#pragma unroll
        for (int kb = 0; kb < KB; ++kb) {
            const uint32_t bar = smem_addr(&bars[kb]);
            const uint32_t sa = sbase + kb * kStage, sb = sa + kAtomA;
            mbar_arrive_expect_tx(bar, kStage);
            tma_load_2d(sa, &tmA, bar, k0 + kb * 64, m0);
            tma_load_2d(sb, &tmB, bar, k0 + kb * 64, 0);
        }
        bool ok = true;
        constexpr uint32_t idesc = idesc_bf16_f32(128, 16);
        for (int kb = 0; kb < KB && ok; ++kb) {
            ok = mbar_wait_bounded(smem_addr(&bars[kb]), 0, flags);
            if (!ok) break;
            tc_fence_after();
            const uint32_t sa = sbase + kb * kStage, sb = sa + kAtomA;
#pragma unroll
            for (int w = 0; w < 4; ++w)
                umma_bf16(tmem, sw128_kmajor_desc(sa + w * 32), sw128_kmajor_desc(sb + w * 32), idesc,
                          (kb | w) ? 1u : 0u);
        }
        if (ok) umma_commit(smem_addr(&bars[KB]));
        s_ok = ok ? 1 : 0;
    }
    __syncthreads();
    bool ok = s_ok != 0;
    if (ok) ok = mbar_wait_bounded(smem_addr(&bars[KB]), 0, flags);
    tc_fence_after();
    if (ok) {
        float r[16];
        tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16), r);
        const int m = m0 + warp * 32 + lane;
        if (m < M) {
#pragma unroll
            for (int n = 0; n < 16; ++n)
                if (n < n_rows) partial[((size_t)split * n_rows + n) * M + m] = r[n];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 32);
}

// act[n][m] = bf16(SiLU(sum_s partial[s][n][m]))
__global__ void silu_reduce_kernel(const float *__restrict__ partial, int splits, int n_rows, int M,
                                   uint16_t *__restrict__ act) {
    griddep_wait();
    griddep_launch_dependents();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_rows * M) return;
    float a = 0.f;
    for (int s = 0; s < splits; ++s) a += partial[(size_t)s * n_rows * M + i];
    const float silu = a / (1.0f + expf(-a));
    act[i] = f32_to_bf16_rne(silu);
}

// out[n][m] = sum_s partial[s][n][m]
__global__ void sum_reduce_kernel(const float *__restrict__ partial, int splits, int n_rows, int M,
                                  float *__restrict__ out) {
    griddep_wait();
    griddep_launch_dependents();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_rows * M) return;
    float a = 0.f;
    for (int s = 0; s < splits; ++s) a += partial[(size_t)s * n_rows * M + i];
    out[i] = a;
}

template <int D, int DP>
cudaError_t launch_pk(const tb_dims &d, const uint16_t *K, const uint16_t *Wk, uint16_t *Kp,
                      const int32_t *tok_begin, const int32_t *tok_count, int32_t max_tok,
                      uint32_t *flags, cudaStream_t st) {
    CUtensorMap mK, mW;
    if (!make_map(&mK, K, D, (uint64_t)d.batch * d.n_kv_heads * d.ctx_cap, 128) ||
        !make_map(&mW, Wk, D, (uint64_t)d.n_kv_heads * DP, DP))
        return cudaErrorInvalidValue;
    constexpr int smem = 1024 + (D / 64) * (kAtomA + DP * 128);
    static std::atomic<int> smem_set[kMaxDevices];
    cudaError_t e = ensure_dynamic_smem((const void *)project_keys_kernel<D, DP>, smem, smem_set);
    if (e != cudaSuccess) return e;
    dim3 grid((max_tok + 127) / 128, d.n_kv_heads, d.batch);
    return launch_pdl(project_keys_kernel<D, DP>, grid, dim3(128), smem, st, mK, mW, Kp, tok_begin, tok_count,
                      d.n_kv_heads, d.ctx_cap, flags);
}

constexpr int kKB = 4;  // 64-wide K blocks per CTA (256 of K)

cudaError_t launch_skinny(const uint16_t *A, const uint16_t *B, float *partial, int M, int K,
                          int n_rows, uint32_t *flags, cudaStream_t st) {
    CUtensorMap mA, mB;
    if (!make_map(&mA, A, K, M, 128) || !make_map(&mB, B, K, n_rows, 16)) return cudaErrorInvalidValue;
    constexpr int smem = 1024 + kKB * (kAtomA + 16 * 128);
    static std::atomic<int> smem_set[kMaxDevices];
    cudaError_t e = ensure_dynamic_smem((const void *)skinny_gemm_kernel<kKB>, smem, smem_set);
    if (e != cudaSuccess) return e;
    return launch_pdl(skinny_gemm_kernel<kKB>, dim3(M / 128, K / (kKB * 64)), dim3(128), smem, st, mA, mB, partial,
                      M, n_rows, flags);
}

struct PredWs {
    uint32_t *flags;
    float *p1;
    uint16_t *act;
    float *p2;
};

PredWs carve_pred(void *ws, int batch, int hidden, int inter, int n_out) {
    uint8_t *p = static_cast<uint8_t *>(ws);
    PredWs w;
    size_t off = kWsHeaderBytes;
    w.flags = reinterpret_cast<uint32_t *>(p);
    w.p1 = reinterpret_cast<float *>(p + off);
    off += align_up((size_t)(hidden / (kKB * 64)) * batch * inter * 4, 256);
    w.act = reinterpret_cast<uint16_t *>(p + off);
    off += align_up((size_t)batch * inter * 2, 256);
    w.p2 = reinterpret_cast<float *>(p + off);
    return w;
}

}  // namespace

size_t predict_ws_bytes(int32_t batch, int32_t hidden, int32_t inter, int32_t n_out) {
    return kWsHeaderBytes + align_up((size_t)(hidden / (kKB * 64)) * batch * inter * 4, 256) +
           align_up((size_t)batch * inter * 2, 256) +
           align_up((size_t)(inter / (kKB * 64)) * batch * n_out * 4, 256);
}

cudaError_t launch_project_keys(const tb_dims &d, const uint16_t *K, const uint16_t *Wk,
                                uint16_t *Kp, const int32_t *tok_begin, const int32_t *tok_count,
                                int32_t max_tok, void *ws, cudaStream_t st) {
    uint32_t *flags = static_cast<uint32_t *>(ws);
    if (d.head_dim == 128)
        return d.d_proj == 32 ? launch_pk<128, 32>(d, K, Wk, Kp, tok_begin, tok_count, max_tok, flags, st)
                              : launch_pk<128, 16>(d, K, Wk, Kp, tok_begin, tok_count, max_tok, flags, st);
    return d.d_proj == 32 ? launch_pk<64, 32>(d, K, Wk, Kp, tok_begin, tok_count, max_tok, flags, st)
                          : launch_pk<64, 16>(d, K, Wk, Kp, tok_begin, tok_count, max_tok, flags, st);
}

cudaError_t launch_predict_queries(const uint16_t *h, const uint16_t *W1, const uint16_t *W2,
                                   float *qp, int32_t batch, int32_t hidden, int32_t inter,
                                   int32_t n_out, void *ws, cudaStream_t st) {
    PredWs w = carve_pred(ws, batch, hidden, inter, n_out);
    cudaError_t e = launch_skinny(W1, h, w.p1, inter, hidden, batch, w.flags, st);
    if (e != cudaSuccess) return e;
    const int n1 = batch * inter;
    e = launch_pdl(silu_reduce_kernel, dim3((n1 + 255) / 256), dim3(256), 0, st, (const float *)w.p1,
                   hidden / (kKB * 64), batch, inter, w.act);
    if (e != cudaSuccess) return e;
    e = launch_skinny(W2, w.act, w.p2, n_out, inter, batch, w.flags, st);
    if (e != cudaSuccess) return e;
    const int n2 = batch * n_out;
    return launch_pdl(sum_reduce_kernel, dim3((n2 + 255) / 256), dim3(256), 0, st, (const float *)w.p2,
                      inter / (kKB * 64), batch, n_out, qp);
}

}  // namespace tb
