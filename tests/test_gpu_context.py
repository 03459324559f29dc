"""Context-parallel selection and attention on one GPU: the ranks' blocks of
one context, run one after another (they never wait on one another, so this is
what separate GPUs compute), with the exchanges emulated by stacking their
tensors.  The merged selection must equal the single-device selection bit for
bit (integer-valued inputs also equal to the oracle's), and the combined
attention output must match the oracle within the attention tolerance."""
import math

import numpy as np
import pytest
import torch

import oracle
import parity
import query_aware_sparse_tb_b200 as tb
import tb_inputs
from query_aware_sparse_tb_b200.decode import ContextShard, DecodeShape, combine_parts, context_blocks

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(integer):
    return tb_inputs.WORKLOADS["llama8k"].scaled(
        name="ctx_par_int" if integer else "ctx_par", batch=2, n_layers=1, n_q_heads=8, n_kv_heads=2,
        head_dim=64 if integer else 128, d_proj=16 if integer else 32, hidden=0, inter=0, producer_stride=1,
        ctx0=0, ctx0_lo=5000, ctx0_hi=7000, sink=16, window=64, budget=300, nbr=1, interval=1, steps=1,
        integer_valued=integer)


@pytest.mark.parametrize("integer,world", [(True, 2), (True, 3), (False, 4)])
def test_context_shards_reproduce_the_single_device_selection(integer, world):
    w = _case(integer)
    T = [t + 1 for t in w.ctx0_per_seq()]
    K, V = tb_inputs.kv_layer(w, 0, DEV)
    Wk = tb_inputs.wk_layer(w, 0, DEV)
    qp = tb_inputs.direct_qp(w, 0, 0, DEV)
    Q = tb_inputs.query(w, 0, 0, DEV)
    cap = w.ctx_cap
    shape = DecodeShape(batch=w.batch, n_layers=1, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                        head_dim=w.head_dim, d_proj=w.d_proj, hidden=0, inter=0, stride=1, sink=w.sink,
                        window=w.window, budget=w.budget, nbr=w.nbr, interval=1, ctx_cap=cap)
    # the single-device selection on the same projected keys
    dm = tb.dims(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.d_proj, cap)
    Kp = torch.zeros(w.batch, w.n_kv_heads, cap, w.d_proj, dtype=torch.bfloat16, device=DEV)
    ws = tb.workspace(256)
    tb.project_keys(dm, K, Wk, Kp, torch.zeros(w.batch, dtype=torch.int32, device=DEV),
                    torch.tensor(T, dtype=torch.int32, device=DEV), cap, ws)
    idx_ref = torch.zeros(w.batch, w.n_q_heads, shape.idx_cap, dtype=torch.int32, device=DEV)
    cnt_ref = torch.zeros(w.batch, w.n_q_heads, dtype=torch.int32, device=DEV)
    bits_ref = torch.zeros(w.batch, w.n_q_heads, shape.words, dtype=torch.int32, device=DEV)
    ws_sel = tb.workspace(tb.score_select_workspace_bytes(dm))
    tb.score_select(dm, qp, w.n_q_heads * w.d_proj, Kp, torch.tensor(T, dtype=torch.int32, device=DEV), w.sink,
                    w.window, w.budget, w.nbr, idx_ref, cnt_ref, bits_ref, ws_sel)
    # the ranks' blocks
    shards = []
    for blk in context_blocks(cap, world, w.window):
        n = blk[1] - blk[0]
        lcap = n + w.window
        Kl = torch.zeros(w.batch, w.n_kv_heads, lcap, w.head_dim, dtype=torch.bfloat16, device=DEV)
        Vl = torch.zeros_like(Kl)
        Kl[:, :, :n] = K[:, :, blk[0]:blk[1]]
        Vl[:, :, :n] = V[:, :, blk[0]:blk[1]]
        sh = ContextShard(shape, blk, Kl, Vl, Wk, DEV)
        sh.project([max(0, min(t, blk[1]) - blk[0]) for t in T])
        shards.append(sh)
    cands = torch.stack([sh.select_local(T, qp).clone() for sh in shards])       # exchange 1
    parts = torch.stack([sh.merge_and_attend(T, cands, Q).clone() for sh in shards])  # exchange 2
    out = torch.empty(w.batch, w.n_q_heads, w.head_dim, device=DEV)
    combine_parts(parts, out)
    torch.cuda.synchronize()
    for sh in shards:
        for x in (sh.ws_sel, sh.ws_attn, sh.ws_small):
            assert tb.workspace_check(x) == 0
        # every rank derives the same global selection, equal to the single-device one
        assert torch.equal(sh.cnt, cnt_ref)
        for b in range(w.batch):
            for h in range(w.n_q_heads):
                n = int(cnt_ref[b, h])
                assert torch.equal(sh.idx[b, h, :n], idx_ref[b, h, :n]), (b, h)
    got = out.cpu().numpy()
    if integer:
        # exact scores: the sets are the oracle's own, and the output is checked
        # against the oracle's attention over them
        Kb, Vb, Qb, Wb = parity.bits16(K), parity.bits16(V), parity.bits16(Q), parity.bits16(Wk)
        qpn = qp.cpu().numpy()
        for b in range(w.batch):
            for h in range(w.n_q_heads):
                Kp_o = oracle.project_keys(Kb[b, h // 4, :T[b]], Wb[h // 4])
                s = oracle.scores(qpn[b, h], Kp_o, w.sink, T[b] - w.window)
                I_o = oracle.select(s, T[b], w.sink, w.window, w.budget, w.nbr)
                assert np.array_equal(idx_ref[b, h, :cnt_ref[b, h]].cpu().numpy(), I_o), (b, h)
                A = oracle.attention_set(T[b], w.sink, w.window, I_o)
                ref = oracle.attention(Qb[b, h], Kb[b, h // 4], Vb[b, h // 4], A, 1 / math.sqrt(w.head_dim))
                parity.assert_close(got[b, h], ref, f"context-parallel out b {b} h {h}")
    else:
        # the single-device attention over the same sets (itself checked against
        # the oracle by the kernel and schedule tests)
        ref = torch.empty_like(out)
        tb.sparse_decode_attn(dm, Q, K, V, torch.tensor(T, dtype=torch.int32, device=DEV), w.sink, w.window,
                              bits_ref, 1 / math.sqrt(w.head_dim), ref, tb.workspace(tb.attn_workspace_bytes(dm)))
        torch.cuda.synchronize()
        parity.assert_close(got, ref.cpu().numpy(), "context-parallel out")
