"""The workspace-free sparse attention entry point, through the C ABI.

It exists for callers that cannot allocate device memory for the call (an
operator boundary that is handed only its inputs and outputs, or a decode
loop that must not call cudaMalloc).  It runs the same kernel on the same
inputs as the workspace entry point, so its output must equal that entry
point's bit for bit, on two calls in a row (the second call reuses the fixed
scratch the first one left behind).  This file is
collected last on purpose."""
import ctypes
import math

import numpy as np
import pytest
import torch

import parity
import tb_inputs
from query_aware_sparse_tb_b200 import _lib


def _case():
    w = tb_inputs.WORKLOADS["llama8k"].scaled(name="noalloc", batch=2, ctx0=5000, ctx0_lo=5000, ctx0_hi=5000,
                                               steps=8)
    ctx = [5007, 1777]
    sets = tb_inputs.selection_sets(w, ctx, 0.25)
    K, V = tb_inputs.kv_layer(w, 0, "cuda")
    Q = tb_inputs.query(w, 0, 0, "cuda")
    W = (w.ctx_cap + 31) // 32
    bits = torch.from_numpy(parity.pack_sets([[s.numpy() for s in hs] for hs in sets], W).view(np.int32)).cuda()
    d = _lib.dims(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.d_proj, w.ctx_cap)
    return w, d, Q, K, V, torch.tensor(ctx, dtype=torch.int32, device="cuda"), bits


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    w, d, Q, K, V, ctx, bits = _case()
    lib = _lib.load()
    scale = 1.0 / math.sqrt(w.head_dim)
    ref = torch.zeros(w.batch, w.n_q_heads, w.head_dim, device="cuda")
    ws = _lib.workspace(_lib.attn_workspace_bytes(d))
    _lib.sparse_decode_attn(d, Q, K, V, ctx, w.sink, w.window, bits, scale, ref, ws)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        st = lib.tb_sparse_decode_attn_noalloc(ctypes.byref(d), Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                               ctx.data_ptr(), w.sink, w.window, bits.data_ptr(), scale,
                                               out.data_ptr(), stream)
        assert st == _lib.TB_OK, lib.tb_last_error()
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"no-alloc call {call} differs from tb_sparse_decode_attn"


@pytest.mark.gpu
def test_noalloc_rejects_dims_beyond_the_fixed_scratch():
    lib = _lib.load()
    big = _lib.dims(16, 32, 8, 128, 32, 32896)       # 128 (sequence, KV head) pairs
    assert lib.tb_attn_workspace_bytes(ctypes.byref(big)) > (4 << 20)
    fake = 1 << 20
    st = lib.tb_sparse_decode_attn_noalloc(ctypes.byref(big), fake, fake, fake, fake, 16, 64, fake, 0.1, fake, None)
    assert st == _lib.TB_ERR_WORKSPACE
    assert b"fixed scratch" in lib.tb_last_error()
