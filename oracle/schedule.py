"""Decode-loop schedule and the whole-path oracle run (test infrastructure only).

Written from the TokenButler summaries, independently of the library's own
schedule code:

* [ja] 技術概要：TokenButler, コアアーキテクチャ: queries are predicted at fixed
  depth-stride producer layers and consumed by the layers that follow; each
  producer call emits G slot-specific queries per head (reading: G = stride,
  slot j serves layer p + j).
* [ja] 最適化, バッチ処理: keys are projected in batches of N tokens, not at every
  step (reading: N is the window size, so every candidate [S, T-N) has a
  projected key).
* [ja] 最適化, 予測間隔と近隣取得: the predictor (and therefore the selection)
  runs once per prediction interval P; the index set is reused in between.
* [ja] 推論戦略: sink and window are recomputed from the current length at every
  step; the importance set is the one from the last prediction.
"""
from __future__ import annotations

import math

import numpy as np

from . import (attention, attention_set, group_scores, predict_queries, project_keys, scores, select,
               select_inclusive)


def is_prediction_step(step: int, interval: int) -> bool:
    return step % interval == 0


def last_prediction_step(step: int, interval: int) -> int:
    return step - step % interval


def producer_of(layer: int, stride: int) -> int:
    return layer - layer % stride


def slot_of(layer: int, stride: int) -> int:
    return layer % stride


def projection_events(ctx0: int, window: int, steps: int):
    """(step, begin) pairs at which a batch of `window` new keys is projected.
    The prefill projects [0, floor(ctx0/N)*N); afterwards a batch is projected
    at step i when the current length T = ctx0 + i + 1 has run N tokens past
    the projected prefix."""
    proj = (ctx0 // window) * window
    events = []
    for i in range(steps):
        T = ctx0 + i + 1
        if T - proj >= window:
            events.append((i, proj))
            proj += window
    return (ctx0 // window) * window, events


def run(w, data, layers, steps, want_attention=True, heads=None, selection="head", seqs=None, attn_steps=None,
        keep=False):
    """Run the oracle over decode steps [0, steps) for the given layers.

    `data` provides host arrays (numpy; bf16 as uint16):
      data.kv(layer) -> (K, V) each [batch][Hkv][ctx_cap][d]
      data.wk(layer) -> [Hkv][d'][d]
      data.mlp(producer) -> (W1, W2)            (predictor workloads)
      data.h(pred_index, producer) -> [batch][hidden]
      data.qp_direct(pred_index, layer) -> [batch][Hq][d'] float32
      data.q(step, layer) -> [batch][Hq][d]
    `selection` is "head" (one importance set per query head, reading R1),
    "group_max" / "group_sum" (one set per KV head from the largest or the
    fp32 sum of the group's head scores, the group-shared variant; every head
    of the group then attends to that set) or "inclusive" (per query head,
    at most `budget` positions after neighbour fetch, the budget-inclusive
    variant).
    `heads` and `seqs` restrict the work to some query heads and sequences
    (the others get None), `attn_steps` to the steps whose attention output is
    computed (default: every step).  With keep=True a prediction step's entry
    also holds what the selection was taken from: "qp" [batch][Hq][d'] (the
    layer's predicted queries), "scores" [b][h] (the fp32 scores of the
    candidates [S, T-N); group scores in the group-shared modes) and "kp"
    {(b, g): K' rows [0, T-N) of KV head g}.
    Returns {(step, layer): {"idx": [[I_bh]], "out": [batch][Hq][d] or None}}.
    """
    assert selection in ("head", "group_max", "group_sum", "inclusive")
    B, Hq, grp = w.batch, w.n_q_heads, w.group
    heads = list(range(Hq)) if heads is None else list(heads)
    seqs = list(range(B)) if seqs is None else list(seqs)
    ctx0 = w.ctx0_per_seq()
    scale = 1.0 / math.sqrt(w.head_dim)
    res = {}
    cur_idx = {}
    kp_cache = {}
    qp_cache = {}
    for layer in layers:
        K, V = data.kv(layer)
        Wk = data.wk(layer)
        for i in range(steps):
            if is_prediction_step(i, w.interval):
                k = i // w.interval
                if w.hidden > 0:
                    p = producer_of(layer, w.producer_stride)
                    if (k, p) not in qp_cache:
                        W1, W2 = data.mlp(p)
                        qp_cache[(k, p)] = predict_queries(data.h(k, p), W1, W2).reshape(
                            B, w.slots, Hq, w.d_proj)
                    qp = qp_cache[(k, p)][:, slot_of(layer, w.producer_stride)]
                else:
                    qp = data.qp_direct(k, layer)
                sets = []
                kept_scores = []
                for b in range(B):
                    T = ctx0[b] + i + 1
                    hi = T - w.window
                    per_head = []
                    per_head_scores = []
                    group_sets = {}
                    group_scores_ = {}
                    for h in range(Hq):
                        if h not in heads or b not in seqs:
                            per_head.append(None)
                            per_head_scores.append(None)
                            continue
                        g = h // grp
                        if selection not in ("head", "inclusive") and g in group_sets:
                            per_head.append(group_sets[g])
                            per_head_scores.append(group_scores_[g])
                            continue
                        if hi > w.sink:
                            key = (layer, b, g)
                            have = kp_cache.get(key)
                            if have is None or have.shape[0] < hi:
                                kp_cache[key] = project_keys(K[b, g, :hi], Wk[g])
                            if selection in ("head", "inclusive"):
                                s = scores(qp[b, h], kp_cache[key], w.sink, hi)
                            else:
                                s = group_scores(qp[b, g * grp:(g + 1) * grp], kp_cache[key], w.sink, hi,
                                                 selection[len("group_"):])
                        else:
                            s = np.zeros(0, np.float32)
                        pick = select_inclusive if selection == "inclusive" else select
                        I = pick(s, T, w.sink, w.window, w.budget, w.nbr)
                        if selection not in ("head", "inclusive"):
                            group_sets[g] = I
                            group_scores_[g] = s
                        per_head.append(I)
                        per_head_scores.append(s)
                    sets.append(per_head)
                    kept_scores.append(per_head_scores)
                cur_idx[layer] = sets
                if keep:
                    kept = {"qp": qp, "scores": kept_scores,
                            "kp": {(b, g): kp_cache[(layer, b, g)][:ctx0[b] + i + 1 - w.window]
                                   for (l_, b, g) in kp_cache if l_ == layer and b in seqs}}
            out = None
            if want_attention and (attn_steps is None or i in attn_steps):
                Q = data.q(i, layer)
                out = np.zeros((B, Hq, w.head_dim), np.float32)
                for b in seqs:
                    T = ctx0[b] + i + 1
                    for h in heads:
                        g = h // grp
                        A = attention_set(T, w.sink, w.window, cur_idx[layer][b][h])
                        out[b, h] = attention(Q[b, h], K[b, g], V[b, g], A, scale)
            res[(i, layer)] = {"idx": cur_idx[layer], "out": out}
            if keep and is_prediction_step(i, w.interval):
                res[(i, layer)].update(kept)
        kp_cache.clear()
    return res
