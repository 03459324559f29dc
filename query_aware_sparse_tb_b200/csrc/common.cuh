// Device helpers shared by the libtb kernels (sm_100a only).
//
// Thin inline-PTX wrappers for cp.async, mbarrier, TMA tiled loads and the
// tcgen05 tensor-core path, plus bf16 unpacking and the workspace flag word.
// Every wait on an mbarrier is bounded by a clock budget: on expiry the kernel
// records TB_FLAG_TIMEOUT in the workspace flag word and carries on to its
// clean-up path instead of spinning forever.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tb.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libtb is built for sm_100a only"
#endif

namespace tb {

constexpr int kWsHeaderBytes = 256;         // flag word + padding at the start of a workspace
constexpr long long kWaitBudgetCycles = 4000000000LL;  // ~2 s at 2 GHz

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------- flags ----

__device__ __forceinline__ void raise_flag(uint32_t *flags, uint32_t bit) {
    if (flags) atomicOr(flags, bit);
}

// Clamp a device-provided context length into [1, cap]; flag if it was outside.
__device__ __forceinline__ int clamp_ctx(int T, int cap, uint32_t *flags, bool report) {
    if (T < 1 || T > cap) {
        if (report) raise_flag(flags, TB_FLAG_CTX_RANGE);
        T = T < 1 ? 1 : cap;
    }
    return T;
}

// ----------------------------------------------------------------- bf16 ----

// A bf16 pair packed in a 32-bit word: element 0 in the low half.
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Round-to-nearest-even fp32 -> bf16 bits (finite inputs).
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
    uint32_t u = __float_as_uint(f);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

// Order-preserving image of an fp32 value in uint32 (larger float -> larger
// key).  -0 is folded onto +0 first so that equal scores give equal keys.
__device__ __forceinline__ uint32_t score_key(float s) {
    uint32_t u = __float_as_uint(s + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// --------------------------------------------------------------- smem ----

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// Atomic add at GPU scope with acquire-release semantics: the releasing
// half publishes every store ordered before it (the calling thread's, and
// other threads' ordered before it by a CTA barrier); the acquiring half
// makes every store published by earlier releases on the same word visible
// to the caller (and, after a CTA barrier, to its CTA).  Returns the old value.
__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t *p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;\n" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// ------------------------------------------------------------ cp.async ----

// 16-byte global->shared copy; when `valid` is false nothing is read and the
// destination is zero-filled.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n)
                 : "memory");
}

// ------------------------------------------------------------ mbarrier ----

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// As mbar_try_wait, but the thread may sleep in hardware for up to
// `suspend_ns` until the phase completes instead of returning at once, so a
// waiting thread issues (almost) nothing on the shared-memory pipe.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t suspend_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(suspend_ns)
        : "memory");
    return ok != 0;
}
// Wait for phase `parity` of the barrier, giving up after `budget` clock
// cycles (default: the library-wide budget).  Returns false (and flags
// TB_FLAG_TIMEOUT) on expiry.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint32_t *flags,
                                                  long long budget = kWaitBudgetCycles) {
    if (mbar_try_wait(bar, parity)) return true;
    long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > budget) {
            raise_flag(flags, TB_FLAG_TIMEOUT);
            return false;
        }
    }
    return true;
}

// ----------------------------------------------------------------- TMA ----

// 2-D tiled bulk tensor load into this CTA's own shared memory only,
// completion counted on `bar` in bytes.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];\n" ::"r"(dst),
        "l"(map), "r"(bar), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
// Order this thread's earlier generic-proxy shared-memory writes before later
// async-proxy (bulk copy) writes to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(map) : "memory");
}

// ------------------------------------------------------------- tcgen05 ----

// Allocate `ncols` TMEM columns (power of two >= 32); the base address is
// written to shared memory at `dst`.  Whole-warp operation.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored in the
// canonical 128-byte-swizzled layout (rows of 128 B, 8-row groups 1024 B
// apart, tile base 1024-byte aligned), as written by a TMA load with
// CU_TENSOR_MAP_SWIZZLE_128B and a 64-element bf16 box width.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);      // start address  [0,14)
    d |= (uint64_t)1u << 16;                       // leading byte offset (unused here) [16,30)
    d |= (uint64_t)(1024u >> 4) << 32;             // stride byte offset: 8 rows x 128 B [32,46)
    d |= (uint64_t)1u << 46;                       // descriptor version for sm_100 [46,48)
    d |= (uint64_t)2u << 61;                       // layout: 128-byte swizzle [61,64)
    return d;
}

// Shared-memory matrix descriptor for an MN-major operand in the canonical
// 128-byte-swizzled layout: 64 consecutive MN elements (128 B) per line, 8
// lines (consecutive K) per 1024-byte atom, K atoms 1024 B apart, MN atoms
// `mn_stride` bytes apart.  A row-major [K][64] bf16 tile written with the
// 128-byte swizzle is exactly one column of such atoms.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t saddr, uint32_t mn_stride) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);               // start address
    d |= (uint64_t)((mn_stride >> 4) & 0x3FFFu) << 16;     // leading byte offset: next MN atom
    d |= (uint64_t)(1024u >> 4) << 32;                      // stride byte offset: next 8 K lines
    d |= (uint64_t)1u << 46;                                // descriptor version for sm_100
    d |= (uint64_t)2u << 61;                                // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor, kind::f16: bf16 A and B (both K-major), fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
    return (1u << 4)                      // D format: fp32
           | (1u << 7)                    // A format: bf16
           | (1u << 10)                   // B format: bf16
           | ((uint32_t)(N >> 3) << 17)   // N / 8
           | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// D(tmem) (+)= A(smem desc) * B(smem desc)^T, issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on `bar` once every previously issued tcgen05.mma of this thread has
// completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
        : "memory");
}

// Each thread of the warp reads its TMEM lane (warp quarter base + lane id),
// 16 consecutive 32-bit columns starting at `taddr`'s column.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16]) {
    uint32_t v[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
          "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    // The wait names the loaded registers so no use can be scheduled above it.
    asm volatile("tcgen05.wait::ld.sync.aligned;\n"
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                   "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                   "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15])
                 :
                 : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = __uint_as_float(v[i]);
}
// As tmem_ld16, 4 and 8 columns.
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float (&r)[4]) {
    uint32_t v[4];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;\n"
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3])
                 :
                 : "memory");
#pragma unroll
    for (int i = 0; i < 4; ++i) r[i] = __uint_as_float(v[i]);
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&r)[8]) {
    uint32_t v[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                   "=r"(v[6]), "=r"(v[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;\n"
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                   "+r"(v[6]), "+r"(v[7])
                 :
                 : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) r[i] = __uint_as_float(v[i]);
}

// ------------------------------------------------- cp.async -> mbarrier ----

// Arrive on `bar` when every cp.async this thread issued so far has landed
// (the barrier's pending count is raised now and dropped on completion, so
// the thread still makes its own regular arrival).
__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }
// Close this thread's current group of cp.async copies; wait until at most N
// of its groups are still in flight (each thread tracks only its own copies).
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// ------------------------------------------- programmatic dependent launch ----

// Wait until every grid this one depends on through a programmatic launch
// edge has completed and its memory operations are visible; returns at once
// when the grid was launched without that attribute.  A kernel launched with
// programmatic stream serialization calls this before its first access to
// memory an earlier kernel may write.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
// Let the next grid in the stream (if launched with programmatic stream
// serialization) be scheduled before this one has finished.
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// Launch `kernel` with programmatic stream serialization: its CTAs may start
// while the previous kernel in the stream is finishing.  Every libtb kernel
// calls griddep_wait() before its first access to global memory, so the
// attribute only moves launch latency and shared-memory set-up off the
// critical path.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

// The same with a thread-block cluster of `cluster` CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, int cluster, size_t smem,
                                      cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

// ------------------------------------------------------------ clusters ----

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
    return r;
}
// Cluster-wide barrier in two halves.  Every thread of every CTA in the
// cluster must arrive; shared-memory writes made before the arrive are
// visible to ld_dsmem reads made after the wait, in any CTA of the cluster.
// A hardware barrier like __syncthreads, not a poll: it completes once all
// threads have arrived, which the kernels guarantee by calling it at the
// same points on every path.
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_sync() {
    cluster_arrive();
    cluster_wait();
}
// 32-bit read of the word at `local` (an address in this CTA's shared memory)
// in the shared memory of cluster CTA `rank` (distributed shared memory).
__device__ __forceinline__ uint32_t ld_dsmem(const void *local, uint32_t rank) {
    uint32_t ra, v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(ra) : "r"(smem_addr(local)), "r"(rank));
    asm volatile("ld.shared::cluster.u32 %0, [%1];\n" : "=r"(v) : "r"(ra) : "memory");
    return v;
}

// Generic address of the word at `local` (in this CTA's shared memory) in the
// shared memory of cluster CTA `rank`; plain loads through it read
// distributed shared memory, and several can be in flight at once.  The
// mapping is ordered after earlier cluster barriers (volatile asm), so loads
// through it are too.
__device__ __forceinline__ const uint32_t *dsmem_ptr(const uint32_t *local, uint32_t rank) {
    uint64_t g;
    asm volatile("mapa.u64 %0, %1, %2;\n" : "=l"(g) : "l"(local), "r"(rank));
    return reinterpret_cast<const uint32_t *>(g);
}

// ------------------------------------------------------ named barriers ----

// Barrier `id` over `n` threads (whole warps) that also returns whether any of
// them passed `v`.
__device__ __forceinline__ bool bar_any(uint32_t id, uint32_t n, bool v) {
    __syncwarp();  // the barrier is warp-aligned: reconverge after per-lane polling
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void bar_named(uint32_t id, uint32_t n) {
    __syncwarp();
    asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}

}  // namespace tb
