"""The oracle's decode-loop schedule and whole-path run (CPU only).

Invariants fixed by the TokenButler summaries ([ja] 推論戦略 and 最適化):
sink and window always attended, projection in batches of N that always cover
the candidates, the selection reused unchanged for a whole prediction interval,
and sparse attention equal to dense attention when the budget covers every
candidate.
"""
import math

import numpy as np
import torch

import oracle
import tb_inputs
from oracle import schedule


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


class HostData:
    """Host-side (numpy) view of a workload, generated on the CPU."""

    def __init__(self, w):
        self.w = w

    def kv(self, layer):
        K, V = tb_inputs.kv_layer(self.w, layer)
        return _bits(K), _bits(V)

    def wk(self, layer):
        return _bits(tb_inputs.wk_layer(self.w, layer))

    def mlp(self, p):
        W1, W2 = tb_inputs.mlp_weights(self.w, p)
        return _bits(W1), _bits(W2)

    def h(self, k, p):
        return _bits(tb_inputs.hidden_state(self.w, k, p))

    def qp_direct(self, k, layer):
        return tb_inputs.direct_qp(self.w, k, layer).numpy()

    def q(self, i, layer):
        return _bits(tb_inputs.query(self.w, i, layer))


def test_projection_events_cover_candidates():
    for ctx0 in (1, 63, 64, 65, 299, 8192, 1000):
        for N in (1, 16, 64):
            proj, events = schedule.projection_events(ctx0, N, 200)
            assert proj % N == 0 and proj <= ctx0 < proj + N
            it = iter(events)
            nxt = next(it, None)
            for i in range(200):
                if nxt is not None and nxt[0] == i:
                    assert nxt[1] == proj
                    proj += N
                    nxt = next(it, None)
                T = ctx0 + i + 1
                assert T - N <= proj, "every candidate [S, T-N) has a projected key"
                assert proj <= T, "only existing tokens are projected"


def test_prediction_schedule():
    assert [i for i in range(40) if schedule.is_prediction_step(i, 16)] == [0, 16, 32]
    assert schedule.last_prediction_step(37, 16) == 32
    assert [schedule.producer_of(l, 4) for l in range(9)] == [0, 0, 0, 0, 4, 4, 4, 4, 8]
    assert [schedule.slot_of(l, 4) for l in range(6)] == [0, 1, 2, 3, 0, 1]


def _small_llama(**kw):
    base = tb_inputs.WORKLOADS["llama8k"].scaled(
        name="llama_small", n_layers=2, n_q_heads=8, n_kv_heads=2, hidden=256, inter=64,
        producer_stride=2, ctx0=700, ctx0_lo=700, ctx0_hi=700, sink=4, window=16,
        budget=40, interval=4, steps=9)
    return base.scaled(**kw)


def test_run_tiny300_invariants():
    w = tb_inputs.WORKLOADS["tiny300"]
    res = schedule.run(w, HostData(w), layers=[0], steps=1)
    r = res[(0, 0)]
    T = w.ctx0 + 1
    assert T == 300
    for h in range(w.n_q_heads):
        I = r["idx"][0][h]
        nC = T - w.window - w.sink
        assert min(w.budget, nC) <= len(I) <= min(3 * w.budget, nC)
        assert np.all(I >= w.sink) and np.all(I < T - w.window)
        assert np.all(np.diff(I) > 0)
    assert np.all(np.isfinite(r["out"]))


def test_run_group_selection_shares_one_set_per_kv_head():
    # the group-shared variant: the 4 heads of a KV head attend to one set, the
    # top-B of the group score (max or fp32 sum of the head scores)
    w = tb_inputs.WORKLOADS["tiny300"]
    data = HostData(w)
    T = w.ctx0 + 1
    K, _ = data.kv(0)
    qp = data.qp_direct(0, 0)
    for red in ("max", "sum"):
        r = schedule.run(w, data, layers=[0], steps=1, selection="group_" + red)[(0, 0)]
        for g in range(w.n_kv_heads):
            Kp = oracle.project_keys(K[0, g, :T - w.window], data.wk(0)[g])
            s = oracle.group_scores(qp[0, 4 * g:4 * g + 4], Kp, w.sink, T - w.window, red)
            want = oracle.select(s, T, w.sink, w.window, w.budget, w.nbr)
            for h in range(4 * g, 4 * g + 4):
                assert np.array_equal(r["idx"][0][h], want), (red, g, h)
        assert np.all(np.isfinite(r["out"]))


def test_run_reuses_selection_over_interval():
    w = _small_llama()
    res = schedule.run(w, HostData(w), layers=[0, 1], steps=w.steps)
    for layer in (0, 1):
        for i in range(w.steps):
            p = schedule.last_prediction_step(i, w.interval)
            for h in range(w.n_q_heads):
                assert np.array_equal(res[(i, layer)]["idx"][0][h], res[(p, layer)]["idx"][0][h])
        # a new prediction (later, longer context) produces a different set somewhere
        assert any(not np.array_equal(res[(4, layer)]["idx"][0][h], res[(0, layer)]["idx"][0][h])
                   for h in range(w.n_q_heads))


def test_run_budget_covering_context_equals_dense():
    w = _small_llama(budget=10_000, steps=2, interval=1)
    data = HostData(w)
    res = schedule.run(w, data, layers=[1], steps=2)
    K, V = data.kv(1)
    scale = 1.0 / math.sqrt(w.head_dim)
    for i in range(2):
        Q = data.q(i, 1)
        T = w.ctx0 + i + 1
        for h in range(w.n_q_heads):
            g = h // w.group
            dense = oracle.attention(Q[0, h], K[0, g], V[0, g], np.arange(T, dtype=np.int32), scale)
            assert np.allclose(res[(i, 1)]["out"][0, h], dense, rtol=1e-6, atol=1e-7)


def test_run_window_follows_current_length_between_predictions():
    # Reading R5: sink and window follow the current length T at every step,
    # the importance set is the one chosen at the last prediction, and tokens
    # that leave the window mid-interval are not added back until the next
    # prediction.  With a budget covering every candidate the set is exactly
    # [S, T_p - N), so the attended rows are [0, T_p - N) U [T - N, T): the
    # rows [T_p - N, T - N) are left out until the next prediction.
    w = _small_llama(budget=10_000, interval=4, steps=6)
    data = HostData(w)
    res = schedule.run(w, data, layers=[0], steps=w.steps)
    K, V = data.kv(0)
    scale = 1.0 / math.sqrt(w.head_dim)
    S, N = w.sink, w.window
    for i in range(w.steps):
        p = schedule.last_prediction_step(i, w.interval)
        T, Tp = w.ctx0 + i + 1, w.ctx0 + p + 1
        A = np.concatenate([np.arange(0, Tp - N), np.arange(T - N, T)]).astype(np.int32)
        assert (i == p) == (A.size == T), "rows leave the attended set only between predictions"
        Q = data.q(i, 0)
        for h in range(w.n_q_heads):
            assert np.array_equal(res[(i, 0)]["idx"][0][h], np.arange(S, Tp - N))
            g = h // w.group
            want = oracle.attention(Q[0, h], K[0, g], V[0, g], A, scale)
            assert np.allclose(res[(i, 0)]["out"][0, h], want, rtol=1e-6, atol=1e-7), (i, h)


def test_run_layer_reads_its_producer_slot():
    # slot j of the producer's G-slot output serves layer p + j (reading R2)
    w = _small_llama(steps=1)
    data = HostData(w)
    res = schedule.run(w, data, layers=[0, 1], steps=1, want_attention=False)
    W1, W2 = data.mlp(0)
    qp = oracle.predict_queries(data.h(0, 0), W1, W2).reshape(w.batch, w.slots, w.n_q_heads, w.d_proj)
    K, _ = data.kv(1)
    T = w.ctx0 + 1
    hi = T - w.window
    Kp = oracle.project_keys(K[0, 0, :hi], data.wk(1)[0])
    sets = [oracle.select(oracle.scores(qp[0, j, 0], Kp, w.sink, hi), T, w.sink, w.window, w.budget, w.nbr)
            for j in range(w.slots)]
    assert not np.array_equal(sets[0], sets[1]), "the two slots must select differently for this check"
    assert np.array_equal(res[(0, 1)]["idx"][0][0], sets[1])


def test_run_inclusive_selection_holds_at_most_budget():
    # the budget-inclusive variant: per head, the importance set after
    # neighbour fetch has at most B positions, is the one orc_select_inclusive
    # gives on that head's scores, and is reused over the interval like any other
    w = _small_llama(interval=4, steps=5)
    data = HostData(w)
    res = schedule.run(w, data, layers=[1], steps=w.steps, selection="inclusive")
    K, _ = data.kv(1)
    W1, W2 = data.mlp(0)
    qp = oracle.predict_queries(data.h(0, 0), W1, W2).reshape(w.batch, w.slots, w.n_q_heads, w.d_proj)[:, 1]
    T = w.ctx0 + 1
    hi = T - w.window
    for h in range(w.n_q_heads):
        Kp = oracle.project_keys(K[0, h // w.group, :hi], data.wk(1)[h // w.group])
        want = oracle.select_inclusive(oracle.scores(qp[0, h], Kp, w.sink, hi), T, w.sink, w.window, w.budget,
                                       w.nbr)
        got = res[(0, 1)]["idx"][0][h]
        assert np.array_equal(got, want), h
        assert 0 < got.size <= w.budget
        for i in range(1, 4):
            assert np.array_equal(res[(i, 1)]["idx"][0][h], got)
    assert np.all(np.isfinite(res[(0, 1)]["out"]))
