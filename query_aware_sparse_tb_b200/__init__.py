"""TokenButler decode-time token selection and sparse attention on B200.

The compute lives in libtb.so (hand-written CUDA for sm_100a, C ABI in
include/tb.h).  This package is the thin Python side: the ctypes binding
(`_lib`), the in-tree build (`build`) and the decode-loop driver (`decode`),
which strings the five entry points together on device-resident buffers.
There is no CPU fallback: every call goes to the CUDA library or raises.
"""
from ._lib import (TbDims, TbError, attn_workspace_bytes, decode_attn, dims, kv_append, load,  # noqa: F401
                   predict_queries, predict_queries_workspace_bytes, project_keys,
                   project_keys_workspace_bytes, score_select, score_select_group, score_select_inclusive,
                   score_select_scores, score_select_workspace_bytes, select_bits_from_idx, sparse_decode_attn,
                   sparse_decode_attn_noalloc, workspace, workspace_check)

__all__ = [
    "TbDims", "TbError", "dims", "load", "workspace", "workspace_check",
    "project_keys", "predict_queries", "score_select", "score_select_group", "score_select_inclusive",
    "score_select_scores", "select_bits_from_idx",
    "sparse_decode_attn", "sparse_decode_attn_noalloc", "decode_attn", "kv_append",
    "attn_workspace_bytes", "score_select_workspace_bytes",
    "predict_queries_workspace_bytes", "project_keys_workspace_bytes",
]
