"""Whole-schedule parity of the CUDA decode loop against the oracle's own
decode loop (oracle/schedule.py), on chosen layers, sequences and query heads.

For every prediction step and checked (layer, sequence, head):
  * q' (the producer MLP's output) within the attention tolerance of the oracle's;
  * every projected key row the selection reads, [0, T-N), against the exact
    product (parity.kprime_matches), including rows projected in batches
    during decoding;
  * the kernel's own fp32 scores (tb_score_select_scores) within a bound of
    the oracle's scores derived from the measured q' and K' differences plus
    the fp32 summation bound;
  * the GPU's set exactly the selection rule's set on the kernel's own scores;
  * the GPU's set equal to the oracle's, or differing only next to candidates
    whose oracle scores are within that bound of the B-th score (and then at
    least two candidates must share that band: a genuine near-tie).
Between predictions the index lists, counts and bitmaps of every layer stay
byte-identical.  At the chosen attention steps every checked head's output is
compared with the oracle's: directly where the GPU's set equals the oracle's,
otherwise by running the GPU attention once more on the oracle's sets (the
GPU stage fed the oracle's inputs); every checked head is compared either way.
Nothing produced by the GPU is ever passed to the oracle.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import parity
import tb_inputs
from oracle import schedule as oschedule
import query_aware_sparse_tb_b200 as tb
from query_aware_sparse_tb_b200.decode import is_prediction_step, producer_layer, query_slot

DEV = "cuda"


def host_kv(run, l):
    """Layer l's K and V as host bf16 bits, from the device or, for an
    offloaded run, from its pinned host cache."""
    dec = run.dec
    if getattr(dec, "offloaded", False):
        return parity.bits16(dec.K_host[l].tensor), parity.bits16(dec.V_host[l].tensor)
    return parity.bits16(dec.K[l]), parity.bits16(dec.V[l])


class RunData:
    """Host copies (numpy, bf16 as uint16) of a bench.Run's device inputs, in
    the form oracle/schedule.py reads them."""

    def __init__(self, run):
        self.run = run

    def kv(self, l):
        return host_kv(self.run, l)

    def wk(self, l):
        return parity.bits16(self.run.Wk[l])

    def mlp(self, p):
        W1, W2 = self.run.mlp[p]
        return parity.bits16(W1), parity.bits16(W2)

    def h(self, k, p):
        return parity.bits16(self.run.h[k][self.run.producers.index(p)])

    def qp_direct(self, k, l):
        return self.run.qp_direct[k][l].cpu().numpy()

    def q(self, i, l):
        return parity.bits16(self.run.Q[i][l])


def score_band(gq, rq, gk_bits, rk_bits):
    """Bound on |GPU fp32 score - oracle fp32 score| per candidate row, from the
    two sides' queries (float [d']) and projected keys (bf16 bits [n][d']):
    |gq - rq|.|gk| + |rq|.|gk - rk| + the GPU's fp32 summation error + the
    oracle's rounding to fp32."""
    gk = parity.bf16_to_f64(gk_bits)
    rk = parity.bf16_to_f64(rk_bits)
    gq = np.asarray(gq, np.float64)
    rq = np.asarray(rq, np.float64)
    return (np.abs(gk) @ np.abs(gq - rq) + np.abs(gk - rk) @ np.abs(rq)
            + (gk.shape[1] + 2) * 2.0 ** -24 * (np.abs(gk) @ np.abs(gq)) + 2.0 ** -24 * (np.abs(rk) @ np.abs(rq)))


def _group_band(selection, bands, gk_bits, gqs):
    if selection == "group_max":
        return np.max(bands, 0)
    # fp32 head-order sum: the heads' bounds plus three fp32 additions on each side
    gk = np.abs(parity.bf16_to_f64(gk_bits))
    absum = sum(gk @ np.abs(np.asarray(q, np.float64)) for q in gqs)
    return np.sum(bands, 0) + 8 * 2.0 ** -24 * absum


def check_schedule(run, layers, steps, seqs, heads, attn_steps, selection="head", data=None, before_step=None):
    """Run `steps` decode steps of bench.Run `run` (eagerly, through the
    library) and check them against the oracle as described above.  `data`
    gives the oracle its inputs (default: the run's own buffers);
    `before_step(i)`, if given, runs right before decode step i (e.g. a cache
    append).  Returns counts of what was checked."""
    w, dec = run.w, run.dec
    s_ = dec.shape
    S, N, Bud, r = w.sink, w.window, w.budget, w.nbr
    group = selection in ("group_max", "group_sum")
    inclusive = selection == "inclusive"
    ctx0 = run.ctx0
    data = data or RunData(run)
    ref = oschedule.run(w, data, layers=layers, steps=steps, heads=heads, seqs=seqs, attn_steps=set(attn_steps),
                        selection=selection, keep=True)
    groups = sorted({hh // w.group for hh in heads})
    K_host = {}
    for l in layers:
        Kl = data.kv(l)[0]
        K_host.update({(l, b, g): Kl[b, g].copy() for b in seqs for g in groups})
        del Kl
    Wk_host = {l: parity.bits16(run.Wk[l]) for l in layers}
    dm = dec.dims
    scores = torch.empty(w.batch, w.n_q_heads, w.ctx_cap, dtype=torch.float32, device=DEV)
    out2 = torch.empty_like(run.out[0])
    scale = 1.0 / math.sqrt(w.head_dim)
    stats = dict(selections=0, exact_sets=0, near_tie_sets=0, outputs=0, reruns=0)
    kept_sel = None
    for i in range(steps):
        Q, h, qd = run.step_inputs(i)
        snap = {}

        def on_select(l, i=i, qd=qd):
            if l not in layers:
                return
            tb.score_select_scores(dm, dec.ws_sel, dec.ctx[i], S, N, scores)
            if w.hidden > 0:
                q_l = dec.qp[producer_layer(l, s_.stride)][:, query_slot(l, s_.stride)]
            else:
                q_l = qd[l]
            snap[l] = (scores.cpu().numpy(), q_l.cpu().numpy(), {b: parity.bits16(dec.Kp[l][b]) for b in seqs})

        if before_step:
            before_step(i)
        dec.step(i, Q, run.out, h=h, qp_direct=qd, on_select=on_select)
        torch.cuda.synchronize()
        for ws in dec.workspaces():
            assert tb.workspace_check(ws) == 0, f"device flag at step {i}"
        now = [(dec.idx[l].clone(), dec.cnt[l].clone(), dec.bits[l].clone()) for l in layers]
        if is_prediction_step(i, w.interval):
            kept_sel = now
        else:
            # reuse across the interval: byte-identical index state in every layer
            for (a1, a2, a3), (b1, b2, b3) in zip(kept_sel, now):
                assert torch.equal(a1, b1) and torch.equal(a2, b2) and torch.equal(a3, b3), f"step {i}"

        if is_prediction_step(i, w.interval):
            for l in layers:
                R = ref[(i, l)]
                g_scores, g_qp, g_kp = snap[l]
                parity.assert_close(g_qp[seqs][:, heads], R["qp"][seqs][:, heads], f"q' step {i} layer {l}")
                idx_l = dec.idx[l].cpu().numpy()
                cnt_l = dec.cnt[l].cpu().numpy()
                for b in seqs:
                    T = ctx0[b] + i + 1
                    hi = T - N
                    checked_k = set()
                    for hh in heads:
                        g = hh // w.group
                        got = idx_l[b, hh, :cnt_l[b, hh]]
                        o_set = R["idx"][b][hh]
                        what = f"step {i} layer {l} b {b} h {hh}"
                        stats["selections"] += 1
                        if hi <= S:
                            assert got.size == 0 and o_set.size == 0, what
                            stats["exact_sets"] += 1
                            continue
                        rk = R["kp"][(b, g)]
                        gk = g_kp[b][g, :hi]
                        if g not in checked_k:
                            # every K' row the selection read, against the exact product
                            parity.kprime_matches(gk, K_host[(l, b, g)][:hi], Wk_host[l][g])
                            checked_k.add(g)
                        if group:
                            hs = range(g * w.group, (g + 1) * w.group)
                            bands = [score_band(g_qp[b, x], R["qp"][b, x], gk[S:], rk[S:]) for x in hs]
                            band = _group_band(selection, bands, gk[S:], [g_qp[b, x] for x in hs])
                            gs = g_scores[b, g * w.group, S:hi]
                        else:
                            band = score_band(g_qp[b, hh], R["qp"][b, hh], gk[S:], rk[S:])
                            gs = g_scores[b, hh, S:hi]
                        s_ref = R["scores"][b][hh]
                        parity.assert_scores_within(gs, s_ref, band, what + ": scores")
                        parity.assert_selection_valid(got, gs, S, Bud, r, what, inclusive)
                        if np.array_equal(got, o_set):
                            stats["exact_sets"] += 1
                            continue
                        stats["near_tie_sets"] += 1
                        if inclusive:
                            # exact on its own scores (above); which near-equal
                            # candidates ended the prefix may differ from the oracle's
                            continue
                        order = np.lexsort((np.arange(s_ref.size), -s_ref.astype(np.float64)))
                        kB = order[min(Bud, s_ref.size) - 1]
                        sB = float(s_ref[kB])
                        tol = parity.SCORE_TIE_TOL * max(1.0, abs(sB))
                        near = np.abs(s_ref.astype(np.float64) - sB) <= band + band[kB] + tol
                        assert near.sum() >= 2, f"{what}: sets differ without a near-tie at the B-th score"
                        exempt = np.nonzero(near)[0] + S
                        for t in np.setxor1d(got, o_set):
                            assert np.any(np.abs(exempt - t) <= r), f"{what}: position {t} differs ({sB})"

        if i in attn_steps:
            for l in layers:
                R = ref[(i, l)]
                got_out = run.out[l].cpu().numpy()
                idx_l = dec.idx[l].cpu().numpy()
                cnt_l = dec.cnt[l].cpu().numpy()
                differs = False
                for b in seqs:
                    for hh in heads:
                        if np.array_equal(idx_l[b, hh, :cnt_l[b, hh]], R["idx"][b][hh]):
                            parity.assert_close(got_out[b, hh], R["out"][b, hh], f"out step {i} layer {l} b {b} h {hh}")
                            stats["outputs"] += 1
                        else:
                            differs = True
                if differs:
                    # the GPU attention on the oracle's sets (the GPU's own sets
                    # for heads and sequences not checked here)
                    sets = [[idx_l[b, hh, :cnt_l[b, hh]] for hh in range(w.n_q_heads)] for b in range(w.batch)]
                    for b in seqs:
                        for hh in heads:
                            sets[b][hh] = R["idx"][b][hh]
                    bits = torch.from_numpy(parity.pack_sets(sets, s_.words).view(np.int32)).to(DEV)
                    tb.sparse_decode_attn(dm, Q[l], dec.K[l], dec.V[l], dec.ctx[i], S, N, bits, scale, out2,
                                          dec.ws_attn)
                    torch.cuda.synchronize()
                    assert tb.workspace_check(dec.ws_attn) == 0
                    o2 = out2.cpu().numpy()
                    for b in seqs:
                        for hh in heads:
                            parity.assert_close(o2[b, hh], R["out"][b, hh], f"out (oracle sets) step {i} layer {l} "
                                                                            f"b {b} h {hh}")
                            stats["outputs"] += 1
                    stats["reruns"] += 1
    return stats


def sampled_heads(w, groups):
    """All query heads of the given KV heads."""
    return [hh for g in groups for hh in range(g * w.group, (g + 1) * w.group)]


def workload(name, **kw):
    return tb_inputs.WORKLOADS[name].scaled(**kw)
