// tb_kv_append: write the token being decoded into the K and V caches of
// every layer in one launch.
//
// TokenButler technical summary (gist.science), "Significance": the full KV
// cache stays resident on the device and attention reads only the kept rows;
// the decode loop therefore appends one K row and one V row per (sequence,
// KV head, layer) at every step, at position T - 1 where T = ctx_len[b]
// counts the token being decoded.  One thread group copies one 16-byte-vector
// row from a packed source into its cache slot, so a step's appends cost one
// launch instead of one strided copy per layer and tensor.
#include "common.cuh"
#include "internal.h"

namespace tb {
namespace {

constexpr int kThreads = 256;

// src: [n_layers][2][batch][Hkv][D] bf16 (0 = K, 1 = V), 16-byte aligned.
// caches: [2 * n_layers] device addresses, K of layer l at 2l, V at 2l + 1.
template <int D>
__global__ void __launch_bounds__(kThreads)
kv_append_kernel(const uint4 *__restrict__ src, const uint64_t *__restrict__ caches,
                 const int32_t *__restrict__ ctx_len, int n_layers, int B, int Hkv, int Tcap,
                 uint32_t *__restrict__ flags) {
    constexpr int V16 = D / 8;  // 16-byte vectors per row
    griddep_wait();
    griddep_launch_dependents();
    const int rows = n_layers * 2 * B * Hkv;
    const int r = blockIdx.x * (kThreads / V16) + threadIdx.x / V16;
    const int c = threadIdx.x % V16;
    if (r >= rows) return;
    const int g = r % Hkv, b = (r / Hkv) % B, kind = (r / (Hkv * B)) % 2, l = r / (Hkv * B * 2);
    const int pos = ctx_len[b] - 1;
    const uint64_t base = caches[2 * l + kind];
    if (pos < 0 || pos >= Tcap) {
        if (c == 0 && g == 0 && l == 0 && kind == 0) raise_flag(flags, TB_FLAG_CTX_RANGE);
        return;
    }
    if (base == 0 || (base & 15u) != 0) {
        if (c == 0) raise_flag(flags, TB_FLAG_BAD_CACHE);
        return;
    }
    uint4 *dst = reinterpret_cast<uint4 *>(base) + (((size_t)b * Hkv + g) * Tcap + pos) * V16;
    dst[c] = src[(size_t)r * V16 + c];
}

// A wait that runs out on purpose: one thread waits on an mbarrier that no
// one ever arrives on, with a short clock budget; the bounded wait gives up,
// raises TB_FLAG_TIMEOUT and the kernel returns.  Checks, on the device, the
// path every pipeline wait takes when a peer stops making progress.
__global__ void bounded_wait_selftest_kernel(uint32_t *flags, long long budget) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_addr(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_mbar_init();
        (void)mbar_wait_bounded(b, 0, flags, budget);
    }
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(void *ws, long long budget_cycles, cudaStream_t st) {
    bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(static_cast<uint32_t *>(ws), budget_cycles);
    return cudaGetLastError();
}

cudaError_t launch_kv_append(const tb_dims &d, int32_t n_layers, const uint16_t *src, const uint64_t *caches,
                             const int32_t *ctx_len, void *ws, cudaStream_t st) {
    uint32_t *flags = static_cast<uint32_t *>(ws);
    const int rows = n_layers * 2 * d.batch * d.n_kv_heads;
    const int per_block = kThreads / (d.head_dim / 8);
    const dim3 grid((rows + per_block - 1) / per_block);
    const uint4 *s = reinterpret_cast<const uint4 *>(src);
    if (d.head_dim == 128)
        return launch_pdl(kv_append_kernel<128>, grid, dim3(kThreads), 0, st, s, caches, ctx_len, n_layers, d.batch,
                          d.n_kv_heads, d.ctx_cap, flags);
    return launch_pdl(kv_append_kernel<64>, grid, dim3(kThreads), 0, st, s, caches, ctx_len, n_layers, d.batch,
                      d.n_kv_heads, d.ctx_cap, flags);
}

}  // namespace tb
