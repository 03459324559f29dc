"""Full-size parity on sampled outputs: one layer of each large workload at its
full context and batch (the per-layer launch configuration the benchmark
times), checked stage by stage against the oracle on sampled sequences and KV
heads (the oracle computes those one by one)."""
import math

import numpy as np
import pytest
import torch

import bench
import oracle
import parity
import tb_inputs
import query_aware_sparse_tb_b200 as tb

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("name", ["llama64k", "batch16", "long256k"])
def test_full_size_sampled(name):
    w = tb_inputs.WORKLOADS[name].scaled(n_layers=1)
    run = bench.Run(w, DEV, steps=1)
    dec = run.dec
    dec.prefill()
    Q, h, qd = run.step_inputs(0)
    dec.step(0, Q, run.out, h=h, qp_direct=qd)
    torch.cuda.synchronize()
    for ws in dec.workspaces():
        assert tb.workspace_check(ws) == 0

    ctx0 = run.ctx0
    samples = sorted({(0, 0), (w.batch - 1, w.n_kv_heads - 1)})
    K0, V0 = run.K[0], run.V[0]
    Wk = parity.bits16(run.Wk[0])
    Kp_gpu = dec.Kp[0]

    # (b) predicted queries: the producer's MLP output
    W1, W2 = run.mlp[0]
    qp_ref = oracle.predict_queries(parity.bits16(h[0]), parity.bits16(W1), parity.bits16(W2))
    parity.assert_close(dec.qp[0].reshape(w.batch, -1).cpu().numpy(), qp_ref, f"{name} q'")
    qp_ref = qp_ref.reshape(w.batch, w.slots, w.n_q_heads, w.d_proj)[:, 0]

    Kp_in = Kp_gpu.clone()
    refs = {}
    kp_refs = {}
    for (b, g) in samples:
        T = ctx0[b] + 1
        Kb = parity.bits16(K0[b, g])
        n = dec.prefill_len[b]
        # (a) projected keys of the prefill, against the exact product
        parity.kprime_matches(parity.bits16(Kp_gpu[b, g, :n]), Kb[:n], Wk[g])
        # the oracle's own K' and selection for this (b, g)
        Kp_ref = oracle.project_keys(Kb[:T - w.window], Wk[g])
        Kp_in[b, g, :T - w.window] = parity.from_bits16(Kp_ref)
        kp_refs[(b, g)] = Kp_ref
        for hh in range(4 * g, 4 * g + 4):
            s = oracle.scores(qp_ref[b, hh], Kp_ref, w.sink, T - w.window)
            refs[(b, hh)] = (s, oracle.select(s, T, w.sink, w.window, w.budget, w.nbr))

    # (c) selection, fed the oracle's K' and q': the kernel's own fp32 scores
    # (tb_score_select_scores) within the fp32 bound of the oracle's, its set
    # exactly the rule's set on those scores, and equal to the oracle's set up
    # to near-ties
    dm = dec.dims
    qpt = torch.from_numpy(np.ascontiguousarray(qp_ref)).to(DEV)
    idx = torch.zeros_like(dec.idx[0])
    cnt = torch.zeros_like(dec.cnt[0])
    bits = torch.zeros_like(dec.bits[0])
    scores = torch.empty(w.batch, w.n_q_heads, w.ctx_cap, dtype=torch.float32, device=DEV)

    def gpu_scores(b, h):
        return scores[b, h].cpu().numpy()

    tb.score_select(dm, qpt, w.n_q_heads * w.d_proj, Kp_in, dec.ctx[0], w.sink, w.window, w.budget, w.nbr,
                    idx, cnt, bits, dec.ws_sel)
    tb.score_select_scores(dm, dec.ws_sel, dec.ctx[0], w.sink, w.window, scores)
    torch.cuda.synchronize()
    n_diff = 0
    for (b, hh), (s, ref) in refs.items():
        T = ctx0[b] + 1
        hi = T - w.window
        got = idx[b, hh, :cnt[b, hh]].cpu().numpy()
        gs = gpu_scores(b, hh)[w.sink:hi]
        what = f"{name} b={b} h={hh}"
        parity.assert_scores_within(gs, s, parity.f32_sum_bound(qp_ref[b, hh], kp_refs[(b, hh // 4)][w.sink:hi]),
                                    what)
        parity.assert_selection_valid(got, gs, w.sink, w.budget, w.nbr, what)
        n_diff += parity.assert_sets_match(got, ref, s, w.sink, w.budget, w.nbr, False, what)

    # (c') the group-shared variant (one set per KV head, group max) on the same inputs
    tb.score_select_group(dm, qpt, w.n_q_heads * w.d_proj, Kp_in, dec.ctx[0], w.sink, w.window, w.budget, w.nbr,
                          "max", idx, cnt, bits, dec.ws_sel)
    tb.score_select_scores(dm, dec.ws_sel, dec.ctx[0], w.sink, w.window, scores)
    torch.cuda.synchronize()
    assert tb.workspace_check(dec.ws_sel) == 0
    for (b, g), Kp_ref in kp_refs.items():
        T = ctx0[b] + 1
        hi = T - w.window
        s = oracle.group_scores(qp_ref[b, 4 * g:4 * g + 4], Kp_ref, w.sink, hi, "max")
        ref = oracle.select(s, T, w.sink, w.window, w.budget, w.nbr)
        got = idx[b, 4 * g, :cnt[b, 4 * g]].cpu().numpy()
        what = f"{name} group b={b} g={g}"
        gs = gpu_scores(b, 4 * g)[w.sink:hi]
        bound = np.max([parity.f32_sum_bound(qp_ref[b, h], Kp_ref[w.sink:hi]) for h in range(4 * g, 4 * g + 4)], 0)
        parity.assert_scores_within(gs, s, bound, what)
        parity.assert_selection_valid(got, gs, w.sink, w.budget, w.nbr, what)
        n_diff += parity.assert_sets_match(got, ref, s, w.sink, w.budget, w.nbr, False, what)
        for hh in range(4 * g + 1, 4 * g + 4):
            assert np.array_equal(idx[b, hh, :cnt[b, hh]].cpu().numpy(), got)

    # (c'') the budget-inclusive variant (at most B positions per head after
    # neighbour fetch), same inputs and the same exact checks
    if w.budget <= 8192:
        tb.score_select_inclusive(dm, qpt, w.n_q_heads * w.d_proj, Kp_in, dec.ctx[0], w.sink, w.window, w.budget,
                                  w.nbr, idx, cnt, bits, dec.ws_sel)
        tb.score_select_scores(dm, dec.ws_sel, dec.ctx[0], w.sink, w.window, scores)
        torch.cuda.synchronize()
        assert tb.workspace_check(dec.ws_sel) == 0
        for (b, hh), (s, _) in refs.items():
            T = ctx0[b] + 1
            hi = T - w.window
            got = idx[b, hh, :cnt[b, hh]].cpu().numpy()
            what = f"{name} inclusive b={b} h={hh}"
            assert got.size <= w.budget and np.all(np.diff(got) > 0), what
            gs = gpu_scores(b, hh)[w.sink:hi]
            parity.assert_scores_within(gs, s, parity.f32_sum_bound(qp_ref[b, hh], kp_refs[(b, hh // 4)][w.sink:hi]),
                                        what)
            parity.assert_selection_valid(got, gs, w.sink, w.budget, w.nbr, what, inclusive=True)

    # (d) sparse attention on the oracle's sets, dense attention
    W = dec.shape.words
    sets = [[refs.get((b, hh), (None, np.zeros(0, np.int32)))[1] for hh in range(w.n_q_heads)]
            for b in range(w.batch)]
    bits_ref = torch.from_numpy(parity.pack_sets(sets, W).view(np.int32)).to(DEV)
    out_s = torch.zeros(w.batch, w.n_q_heads, w.head_dim, device=DEV)
    out_d = torch.zeros_like(out_s)
    scale = 1 / math.sqrt(w.head_dim)
    tb.sparse_decode_attn(dm, Q[0], K0, V0, dec.ctx[0], w.sink, w.window, bits_ref, scale, out_s, dec.ws_attn)
    tb.decode_attn(dm, Q[0], K0, V0, dec.ctx[0], scale, out_d, dec.ws_attn)
    torch.cuda.synchronize()
    Qb = parity.bits16(Q[0])
    for (b, hh), (_, ref) in refs.items():
        g = hh // 4
        T = ctx0[b] + 1
        Kb, Vb = parity.bits16(K0[b, g, :T]), parity.bits16(V0[b, g, :T])
        A = oracle.attention_set(T, w.sink, w.window, ref)
        parity.assert_close(out_s[b, hh].cpu().numpy(), oracle.attention(Qb[b, hh], Kb, Vb, A, scale),
                            f"{name} sparse b={b} h={hh}")
        parity.assert_close(out_d[b, hh].cpu().numpy(),
                            oracle.attention(Qb[b, hh], Kb, Vb, np.arange(T, dtype=np.int32), scale),
                            f"{name} dense b={b} h={hh}")
    assert n_diff <= 8, f"{n_diff} near-tie differences"
