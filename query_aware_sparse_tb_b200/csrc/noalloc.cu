// tb_sparse_decode_attn_noalloc: the sparse decode attention of
// tb_sparse_decode_attn without a caller-provided workspace.
//
// Who needs it: callers that are handed only their input and output buffers
// and have no way to obtain device memory for the call — for example a plugin
// or custom-operator boundary of a serving framework that owns every
// allocation and forbids allocating inside the operator — and decode loops
// that must not call cudaMalloc on the hot path, because cudaMalloc can
// synchronise the whole device and stall every stream.
//
// How: the attention kernel's scratch (per-(sequence, KV head) tickets and
// the partial softmax states of the context slices) lives in one file-scope
// static device array of kNoAllocScratchBytes, which every GPU that loads the
// library keeps until the process exits.  The first call on a device looks up
// that device's address of the array with cudaGetSymbolAddress and clears it
// (a synchronous cudaMemset); that first call must therefore come before any
// stream capture.  Later calls only launch.  Nothing here calls cudaMalloc,
// cudaFree or any allocating library routine.
//
// Sharing: every call on a device uses the same scratch.  The kernel leaves
// its tickets at zero when it finishes, so consecutive calls need no clearing,
// but calls that overlap on the GPU (different streams, or different host
// threads without ordering between them) race on the scratch and produce
// wrong outputs.
#include <cuda_runtime.h>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = TB_NOALLOC_SCRATCH_BYTES;
using tb::kMaxDevices;

// The scratch itself (zero at module load).
static __device__ __align__(256) unsigned char tb_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void *g_scratch[kMaxDevices] = {};

// This device's address of the scratch array, set up (and cleared) on first use.
tb_status scratch_for_current_device(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        tb::set_error("tb_sparse_decode_attn_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
        return TB_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        tb::set_error("tb_sparse_decode_attn_noalloc: device %d beyond the supported %d", dev, kMaxDevices);
        return TB_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, tb_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            tb::set_error("tb_sparse_decode_attn_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
            return TB_ERR_CUDA;
        }
        // a memset of device memory may return before it is done, and the
        // caller's stream need not be ordered after the legacy stream
        e = cudaMemset(p, 0, kNoAllocScratchBytes);
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
        if (e != cudaSuccess) {
            tb::set_error("tb_sparse_decode_attn_noalloc: clearing the scratch: %s", cudaGetErrorString(e));
            return TB_ERR_CUDA;
        }
        g_scratch[dev] = p;
    }
    *out = g_scratch[dev];
    return TB_OK;
}

}  // namespace

extern "C" tb_status tb_sparse_decode_attn_noalloc(const tb_dims *dims, const tb_bf16 *Q, const tb_bf16 *K,
                                                   const tb_bf16 *V, const int32_t *ctx_len, int32_t sink,
                                                   int32_t window, const uint32_t *sel_bits, float scale,
                                                   float *out, void *stream) {
    const char *fn = "tb_sparse_decode_attn_noalloc";
    // the checks of tb_sparse_decode_attn, so both entry points accept the same dims
    tb_status st = tb::check_attn_args(fn, dims, Q, K, V, ctx_len, scale, out, true, sel_bits, sink, window);
    if (st != TB_OK) return st;
    const size_t need = tb::attn_ws_bytes(*dims);
    if (need > kNoAllocScratchBytes) {
        tb::set_error("%s: these dims need %zu bytes of scratch but the fixed scratch holds %zu; "
                      "use tb_sparse_decode_attn with a workspace", fn, need, kNoAllocScratchBytes);
        return TB_ERR_WORKSPACE;
    }
    void *ws = nullptr;
    if ((st = scratch_for_current_device(&ws)) != TB_OK) return st;
    cudaError_t e = tb::launch_attn(*dims, Q, K, V, ctx_len, sink, window, sel_bits, true, scale, out, ws,
                                    (cudaStream_t)stream);
    if (e != cudaSuccess) {
        tb::set_error("%s: %s", fn, cudaGetErrorString(e));
        return TB_ERR_CUDA;
    }
    return TB_OK;
}
