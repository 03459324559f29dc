"""ctypes binding of libtb.so (argument marshalling only).

Every function here converts torch tensors into device pointers and sizes and
calls the C entry point of the same name; all computation happens in the CUDA
kernels behind it.  There is no fallback: if the library is missing or a call
fails, a TbError is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtb.so")

TB_ABI_VERSION = 10
TB_OK, TB_ERR_INVALID_ARG, TB_ERR_UNSUPPORTED, TB_ERR_CUDA, TB_ERR_WORKSPACE, TB_ERR_DEVICE_FLAG = range(6)
TB_FLAG_CTX_RANGE, TB_FLAG_TIMEOUT, TB_FLAG_IDX_OVERFLOW, TB_FLAG_BAD_CACHE = 0x1, 0x2, 0x4, 0x8
TB_GROUP_REDUCE = {"max": 0, "sum": 1}
TB_ATTN_WAIT_ALL, TB_ATTN_PREFETCH_KV = 0, 1
TB_SELECT_AUTO, TB_SELECT_MULTI_KERNEL, TB_SELECT_CLUSTER = 0, 1, 2
TB_ATTN_PLAN_STRIDE = 65

EXPORTS = [
    "tb_abi_version", "tb_status_str", "tb_last_error",
    "tb_score_select_workspace_bytes", "tb_attn_workspace_bytes",
    "tb_predict_queries_workspace_bytes", "tb_project_keys_workspace_bytes",
    "tb_workspace_init", "tb_workspace_check",
    "tb_project_keys", "tb_predict_queries", "tb_score_select", "tb_score_select_group", "tb_score_select_inclusive",
    "tb_score_select_scores", "tb_select_bits_from_idx",
    "tb_select_export_candidates", "tb_select_merge_candidates", "tb_sparse_decode_attn_partial", "tb_attn_combine",
    "tb_sparse_decode_attn", "tb_decode_attn", "tb_sparse_decode_attn_noalloc", "tb_kv_append",
    "tb_selftest_bounded_wait", "tb_attn_set_launch_mode", "tb_attn_launch_mode",
    "tb_select_set_algorithm", "tb_select_algorithm", "tb_attn_plan", "tb_sparse_decode_attn_planned",
]


class TbError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


class TbDims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("d_proj", ctypes.c_int32), ("ctx_cap", ctypes.c_int32)]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libtb.so (it must have been built; nothing is compiled here)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise TbError(-1, f"{path} is missing: build it with `python -m query_aware_sparse_tb_b200.build`")
    lib = ctypes.CDLL(path)
    P, i32, i64, sz, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    D = ctypes.POINTER(TbDims)
    sig = {
        "tb_abi_version": ([], i32),
        "tb_status_str": ([ctypes.c_int], ctypes.c_char_p),
        "tb_last_error": ([], ctypes.c_char_p),
        "tb_score_select_workspace_bytes": ([D], sz),
        "tb_attn_workspace_bytes": ([D], sz),
        "tb_predict_queries_workspace_bytes": ([i32, i32, i32, i32], sz),
        "tb_project_keys_workspace_bytes": ([], sz),
        "tb_workspace_init": ([P, sz, P], ctypes.c_int),
        "tb_workspace_check": ([P, sz, ctypes.POINTER(ctypes.c_uint32), P], ctypes.c_int),
        "tb_project_keys": ([D, P, P, P, P, P, i32, P, sz, P], ctypes.c_int),
        "tb_predict_queries": ([P, P, P, P, i32, i32, i32, i32, P, sz, P], ctypes.c_int),
        "tb_score_select": ([D, P, i64, P, P, i32, i32, i32, i32, P, i32, P, P, P, sz, P], ctypes.c_int),
        "tb_score_select_group": ([D, P, i64, P, P, i32, i32, i32, i32, i32, P, i32, P, P, P, sz, P],
                                  ctypes.c_int),
        "tb_score_select_inclusive": ([D, P, i64, P, P, i32, i32, i32, i32, P, i32, P, P, P, sz, P], ctypes.c_int),
        "tb_score_select_scores": ([D, P, sz, P, i32, i32, P, P], ctypes.c_int),
        "tb_select_bits_from_idx": ([D, P, i32, P, P, P], ctypes.c_int),
        "tb_select_export_candidates": ([D, P, sz, P, i32, P, i32, i32, P, P], ctypes.c_int),
        "tb_select_merge_candidates": ([D, P, i32, i32, P, i32, i32, i32, P, i32, P, i32, i32, i32, P, P, sz, P],
                                       ctypes.c_int),
        "tb_sparse_decode_attn_partial": ([D, P, P, P, P, P, f32, P, P, sz, P], ctypes.c_int),
        "tb_attn_combine": ([P, i32, i32, i32, i32, P, P], ctypes.c_int),
        "tb_sparse_decode_attn": ([D, P, P, P, P, i32, i32, P, f32, P, P, sz, P], ctypes.c_int),
        "tb_sparse_decode_attn_planned": ([D, P, P, P, P, i32, i32, P, P, f32, P, P, sz, P], ctypes.c_int),
        "tb_attn_plan": ([D, P, P, i32, i32, P, P, sz, P], ctypes.c_int),
        "tb_decode_attn": ([D, P, P, P, P, f32, P, P, sz, P], ctypes.c_int),
        "tb_sparse_decode_attn_noalloc": ([D, P, P, P, P, i32, i32, P, f32, P, P], ctypes.c_int),
        "tb_kv_append": ([D, i32, P, P, P, P, sz, P], ctypes.c_int),
        "tb_selftest_bounded_wait": ([P, sz, i64, P], ctypes.c_int),
        "tb_attn_set_launch_mode": ([i32], ctypes.c_int),
        "tb_attn_launch_mode": ([], i32),
        "tb_select_set_algorithm": ([i32], ctypes.c_int),
        "tb_select_algorithm": ([], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    # the signatures above are those of this ABI version; a library built from
    # other sources would be called with the wrong arguments
    if lib.tb_abi_version() != TB_ABI_VERSION:
        raise TbError(-1, f"{path} has ABI version {lib.tb_abi_version()}, this binding needs {TB_ABI_VERSION}: "
                          "rebuild it with `python -m query_aware_sparse_tb_b200.build`")
    if path == LIB_PATH:
        _lib = lib
    return lib


def _check(status: int) -> None:
    if status != TB_OK:
        raise TbError(status, load().tb_last_error().decode())


def _ptr(t) -> int:
    if t is None:
        return 0
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise TbError(TB_ERR_INVALID_ARG, "libtb takes device tensors")
    if not t.is_contiguous():
        raise TbError(TB_ERR_INVALID_ARG, "libtb takes contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def dims(batch, n_q_heads, n_kv_heads, head_dim, d_proj, ctx_cap) -> TbDims:
    return TbDims(batch, n_q_heads, n_kv_heads, head_dim, d_proj, ctx_cap)


def _bytes(t) -> int:
    return t.numel() * t.element_size()


# ------------------------------------------------------------------ workspaces

def score_select_workspace_bytes(d: TbDims) -> int:
    return load().tb_score_select_workspace_bytes(ctypes.byref(d))


def attn_workspace_bytes(d: TbDims) -> int:
    return load().tb_attn_workspace_bytes(ctypes.byref(d))


def predict_queries_workspace_bytes(batch, hidden, inter, n_out) -> int:
    return load().tb_predict_queries_workspace_bytes(batch, hidden, inter, n_out)


def project_keys_workspace_bytes() -> int:
    return load().tb_project_keys_workspace_bytes()


def workspace(nbytes: int, device="cuda", stream=None) -> torch.Tensor:
    """A zero-initialised workspace tensor of at least `nbytes` bytes."""
    if nbytes <= 0:
        raise TbError(TB_ERR_INVALID_ARG, "workspace size must be positive (invalid dims?)")
    ws = torch.empty((nbytes + 255) // 256 * 256, dtype=torch.uint8, device=device)
    _check(load().tb_workspace_init(_ptr(ws), _bytes(ws), _stream(stream)))
    return ws


def workspace_check(ws: torch.Tensor, stream=None) -> int:
    """Return the device flag word (and clear it); 0 means no condition was seen."""
    flags = ctypes.c_uint32(0)
    st = load().tb_workspace_check(_ptr(ws), _bytes(ws), ctypes.byref(flags), _stream(stream))
    if st not in (TB_OK, TB_ERR_DEVICE_FLAG):
        _check(st)
    return flags.value


# ------------------------------------------------------------------ entry points

def project_keys(d: TbDims, K, Wk, Kp, tok_begin, tok_count, max_tok: int, ws, stream=None):
    _check(load().tb_project_keys(ctypes.byref(d), _ptr(K), _ptr(Wk), _ptr(Kp), _ptr(tok_begin),
                                  _ptr(tok_count), int(max_tok), _ptr(ws), _bytes(ws), _stream(stream)))


def predict_queries(h, W1, W2, qp, ws, stream=None):
    batch, hidden = h.shape
    inter = W1.shape[0]
    n_out = W2.shape[0]
    _check(load().tb_predict_queries(_ptr(h), _ptr(W1), _ptr(W2), _ptr(qp), batch, hidden, inter, n_out,
                                     _ptr(ws), _bytes(ws), _stream(stream)))


def score_select(d: TbDims, qp, qp_batch_stride: int, Kp, ctx_len, sink: int, window: int, budget: int,
                 nbr: int, idx, count, sel_bits, ws, stream=None):
    idx_cap = idx.shape[-1]
    _check(load().tb_score_select(ctypes.byref(d), _ptr(qp), int(qp_batch_stride), _ptr(Kp), _ptr(ctx_len),
                                  sink, window, budget, nbr, _ptr(idx), idx_cap, _ptr(count), _ptr(sel_bits),
                                  _ptr(ws), _bytes(ws), _stream(stream)))


def score_select_group(d: TbDims, qp, qp_batch_stride: int, Kp, ctx_len, sink: int, window: int, budget: int,
                       nbr: int, reduce: str, idx, count, sel_bits, ws, stream=None):
    """tb_score_select_group: one set per KV head from the max or sum of the
    group's head scores, written to each of the group's 4 head rows."""
    idx_cap = idx.shape[-1]
    _check(load().tb_score_select_group(ctypes.byref(d), _ptr(qp), int(qp_batch_stride), _ptr(Kp), _ptr(ctx_len),
                                        sink, window, budget, nbr, TB_GROUP_REDUCE[reduce], _ptr(idx), idx_cap,
                                        _ptr(count), _ptr(sel_bits), _ptr(ws), _bytes(ws), _stream(stream)))


def score_select_inclusive(d: TbDims, qp, qp_batch_stride: int, Kp, ctx_len, sink: int, window: int,
                           budget: int, nbr: int, idx, count, sel_bits, ws, stream=None):
    """tb_score_select_inclusive: per head, the importance buffer holds at most
    `budget` positions after neighbour fetch."""
    idx_cap = idx.shape[-1]
    _check(load().tb_score_select_inclusive(ctypes.byref(d), _ptr(qp), int(qp_batch_stride), _ptr(Kp),
                                            _ptr(ctx_len), sink, window, budget, nbr, _ptr(idx), idx_cap,
                                            _ptr(count), _ptr(sel_bits), _ptr(ws), _bytes(ws), _stream(stream)))


def score_select_scores(d: TbDims, ws, ctx_len, sink: int, window: int, scores, stream=None):
    """tb_score_select_scores: the fp32 scores the last selection on `ws` ranked
    ([batch][Hq][ctx_cap] float32; NaN outside the candidates)."""
    _check(load().tb_score_select_scores(ctypes.byref(d), _ptr(ws), _bytes(ws), _ptr(ctx_len), sink, window,
                                         _ptr(scores), _stream(stream)))


def select_export_candidates(d: TbDims, ws, idx, count, budget: int, pos_offset: int, cand, stream=None):
    """tb_select_export_candidates: a rank's top-B (a selection with nbr = 0)
    as (score key, global position) composites, cand [batch][Hq][budget] int64."""
    _check(load().tb_select_export_candidates(ctypes.byref(d), _ptr(ws), _bytes(ws), _ptr(idx), idx.shape[-1],
                                              _ptr(count), int(budget), int(pos_offset), _ptr(cand), _stream(stream)))


def select_merge_candidates(d: TbDims, cand, n_ranks: int, budget: int, ctx_len, sink: int, window: int, nbr: int,
                            idx, count, shard_begin: int, shard_len: int, local_bits, local_cap: int, ws,
                            stream=None):
    """tb_select_merge_candidates: the global selection from every rank's
    candidates, and this rank's attended-row bitmap."""
    _check(load().tb_select_merge_candidates(ctypes.byref(d), _ptr(cand), int(n_ranks), int(budget), _ptr(ctx_len),
                                             sink, window, nbr, _ptr(idx), idx.shape[-1], _ptr(count),
                                             int(shard_begin), int(shard_len), int(local_cap), _ptr(local_bits),
                                             _ptr(ws), _bytes(ws), _stream(stream)))


def sparse_decode_attn_partial(d: TbDims, Q, K, V, rows, bits, scale: float, part, ws, stream=None):
    """tb_sparse_decode_attn_partial: unnormalised attention state over the
    rows of `bits` (part [batch][Hq][d+2] float32)."""
    _check(load().tb_sparse_decode_attn_partial(ctypes.byref(d), _ptr(Q), _ptr(K), _ptr(V), _ptr(rows), _ptr(bits),
                                                float(scale), _ptr(part), _ptr(ws), _bytes(ws), _stream(stream)))


def attn_combine(parts, out, stream=None):
    """tb_attn_combine: parts [n][batch][Hq][d+2] -> out [batch][Hq][d]."""
    n, batch, hq, dd = parts.shape
    _check(load().tb_attn_combine(_ptr(parts), n, batch, hq, dd - 2, _ptr(out), _stream(stream)))


def select_bits_from_idx(d: TbDims, idx, count, sel_bits, stream=None):
    _check(load().tb_select_bits_from_idx(ctypes.byref(d), _ptr(idx), idx.shape[-1], _ptr(count),
                                          _ptr(sel_bits), _stream(stream)))


def sparse_decode_attn(d: TbDims, Q, K, V, ctx_len, sink: int, window: int, sel_bits, scale: float, out, ws,
                       stream=None):
    _check(load().tb_sparse_decode_attn(ctypes.byref(d), _ptr(Q), _ptr(K), _ptr(V), _ptr(ctx_len), sink,
                                        window, _ptr(sel_bits), float(scale), _ptr(out), _ptr(ws), _bytes(ws),
                                        _stream(stream)))


def attn_plan(d: TbDims, sel_bits, ctx_len, sink: int, window: int, plan, ws, stream=None):
    """tb_attn_plan: slice cuts at equal shares of the kept rows,
    plan [batch][Hkv][TB_ATTN_PLAN_STRIDE] int32."""
    _check(load().tb_attn_plan(ctypes.byref(d), _ptr(sel_bits), _ptr(ctx_len), sink, window, _ptr(plan), _ptr(ws),
                               _bytes(ws), _stream(stream)))


def sparse_decode_attn_planned(d: TbDims, Q, K, V, ctx_len, sink: int, window: int, sel_bits, plan, scale: float,
                               out, ws, stream=None):
    """tb_sparse_decode_attn over the slices of a tb_attn_plan."""
    _check(load().tb_sparse_decode_attn_planned(ctypes.byref(d), _ptr(Q), _ptr(K), _ptr(V), _ptr(ctx_len), sink,
                                                window, _ptr(sel_bits), _ptr(plan), float(scale), _ptr(out), _ptr(ws),
                                                _bytes(ws), _stream(stream)))


def sparse_decode_attn_noalloc(d: TbDims, Q, K, V, ctx_len, sink: int, window: int, sel_bits, scale: float,
                               out, stream=None):
    """tb_sparse_decode_attn with the library's fixed scratch instead of a
    workspace (for callers that cannot allocate; see include/tb.h)."""
    _check(load().tb_sparse_decode_attn_noalloc(ctypes.byref(d), _ptr(Q), _ptr(K), _ptr(V), _ptr(ctx_len), sink,
                                                window, _ptr(sel_bits), float(scale), _ptr(out), _stream(stream)))


def attn_set_launch_mode(mode: int):
    """tb_attn_set_launch_mode for the calling thread (TB_ATTN_WAIT_ALL or
    TB_ATTN_PREFETCH_KV; see include/tb.h for the contract of the latter)."""
    _check(load().tb_attn_set_launch_mode(int(mode)))


def select_set_algorithm(algorithm: int):
    """tb_select_set_algorithm for the calling thread (TB_SELECT_AUTO,
    TB_SELECT_MULTI_KERNEL or TB_SELECT_CLUSTER; the result is the same)."""
    _check(load().tb_select_set_algorithm(int(algorithm)))


def decode_attn(d: TbDims, Q, K, V, ctx_len, scale: float, out, ws, stream=None):
    _check(load().tb_decode_attn(ctypes.byref(d), _ptr(Q), _ptr(K), _ptr(V), _ptr(ctx_len), float(scale),
                                 _ptr(out), _ptr(ws), _bytes(ws), _stream(stream)))


def kv_append(d: TbDims, n_layers: int, src, caches, ctx_len, ws, stream=None):
    """tb_kv_append: src [n_layers][2][batch][Hkv][d] bf16 rows of the token
    being decoded; caches an int64 device tensor of the 2*n_layers cache base
    addresses (K of layer l at 2l, V at 2l+1)."""
    _check(load().tb_kv_append(ctypes.byref(d), int(n_layers), _ptr(src), _ptr(caches), _ptr(ctx_len), _ptr(ws),
                               _bytes(ws), _stream(stream)))


def selftest_bounded_wait(ws, budget_cycles: int, stream=None):
    """tb_selftest_bounded_wait: a wait that runs out on purpose (raises TB_FLAG_TIMEOUT in ws)."""
    _check(load().tb_selftest_bounded_wait(_ptr(ws), _bytes(ws), int(budget_cycles), _stream(stream)))
