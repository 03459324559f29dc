"""The two routes of tb_score_select / tb_score_select_group
(tb_select_set_algorithm): the one-kernel cluster path and the multi-kernel
path rank the same fp32 scores and must give the same index lists, counts,
bitmaps and exported scores, bit for bit.  The selection tests against the
oracle run the default route (the cluster kernel wherever it applies), so
these cases keep the multi-kernel route, which long contexts and the
budget-inclusive variant still take, checked against it."""
import numpy as np
import pytest
import torch

import query_aware_sparse_tb_b200 as tb
from query_aware_sparse_tb_b200 import _lib

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(seed, batch, hkv, dp, cap, kind):
    g = torch.Generator().manual_seed(seed)
    hq = 4 * hkv
    if kind == "normal":
        Kp = torch.randn(batch, hkv, cap, dp, generator=g).to(torch.bfloat16)
        qp = torch.randn(batch, hq, dp, generator=g)
    elif kind == "integer":  # small integers: many exactly equal scores
        Kp = torch.randint(-2, 3, (batch, hkv, cap, dp), generator=g).to(torch.bfloat16)
        qp = torch.randint(-1, 2, (batch, hq, dp), generator=g).float()
    elif kind == "coarse":  # integer scores over a few hundred values: ties inside the B-th key's bin
        Kp = torch.randint(-8, 9, (batch, hkv, cap, dp), generator=g).to(torch.bfloat16)
        qp = torch.randint(-3, 4, (batch, hq, dp), generator=g).float()
    elif kind == "outlier":  # a few huge scores squeeze the rest into the lowest score bins
        Kp = torch.randn(batch, hkv, cap, dp, generator=g)
        rows = torch.randint(0, cap, (batch, hkv, 3), generator=g)
        Kp.scatter_(2, rows[..., None].expand(-1, -1, -1, dp), 3e4)
        Kp = Kp.to(torch.bfloat16)
        qp = torch.randn(batch, hq, dp, generator=g).abs()
    else:  # all scores zero: every candidate ties
        Kp = torch.zeros(batch, hkv, cap, dp, dtype=torch.bfloat16)
        qp = torch.randn(batch, hq, dp, generator=g)
    return Kp.to(DEV), qp.to(DEV)


def _run(algo, dm, Kp, qp, ctx, sink, window, budget, nbr, reduce):
    hq, W = dm.n_q_heads, (dm.ctx_cap + 31) // 32
    cap = min((2 * nbr + 1) * budget, dm.ctx_cap)
    idx = torch.full((dm.batch, hq, cap), -7, dtype=torch.int32, device=DEV)
    cnt = torch.full((dm.batch, hq), -7, dtype=torch.int32, device=DEV)
    bits = torch.full((dm.batch, hq, W), -1, dtype=torch.int32, device=DEV)
    scores = torch.empty((dm.batch, hq, dm.ctx_cap), dtype=torch.float32, device=DEV)
    ws = tb.workspace(tb.score_select_workspace_bytes(dm))
    ctx_t = torch.tensor(ctx, dtype=torch.int32, device=DEV)
    _lib.select_set_algorithm(algo)
    try:
        if reduce is None:
            tb.score_select(dm, qp, hq * dm.d_proj, Kp, ctx_t, sink, window, budget, nbr, idx, cnt, bits, ws)
        else:
            tb.score_select_group(dm, qp, hq * dm.d_proj, Kp, ctx_t, sink, window, budget, nbr, reduce, idx, cnt,
                                  bits, ws)
    finally:
        _lib.select_set_algorithm(_lib.TB_SELECT_AUTO)
    tb.score_select_scores(dm, ws, ctx_t, sink, window, scores)
    torch.cuda.synchronize()
    assert tb.workspace_check(ws) == 0
    return idx.cpu().numpy(), cnt.cpu().numpy(), bits.cpu().numpy(), scores.cpu().numpy()


CASES = {
    # name: (batch, Hkv, d', ctx_cap, ctx per sequence, sink, window, budget, nbr)
    "tiny_d16": (1, 2, 16, 384, [299], 4, 16, 32, 1),
    "ragged_modes": (4, 2, 32, 3000, [2999, 20, 150, 1500], 16, 64, 64, 2),
    "tail_not_whole_word": (2, 1, 32, 1000, [999, 517], 3, 5, 100, 3),
    "budget_one_nbr0": (2, 2, 16, 700, [700, 333], 0, 1, 1, 0),
    "llama64k_layer": (1, 8, 32, 65536 + 256, [65537], 16, 64, 8192, 1),
    "batch16_ragged": (16, 8, 32, 32768 + 256, None, 16, 64, 2048, 1),
}


@pytest.mark.parametrize("reduce", [None, "max", "sum"])
@pytest.mark.parametrize("kind", ["normal", "integer", "zeros", "coarse", "outlier"])
@pytest.mark.parametrize("case", list(CASES))
def test_cluster_and_multi_kernel_routes_agree_bit_for_bit(case, kind, reduce):
    batch, hkv, dp, cap, ctx, sink, window, budget, nbr = CASES[case]
    if case in ("llama64k_layer", "batch16_ragged") and kind == "zeros" and reduce is not None:
        pytest.skip("all-ties at full size: covered per head")
    if case == "batch16_ragged" and kind in ("coarse", "outlier") and reduce == "sum":
        pytest.skip("covered by the per-head and max cases")
    if ctx is None:
        ctx = torch.randint(16384, 32769, (batch,), generator=torch.Generator().manual_seed(5)).tolist()
    dm = tb.dims(batch=batch, n_q_heads=4 * hkv, n_kv_heads=hkv, head_dim=128, d_proj=dp, ctx_cap=cap)
    Kp, qp = _inputs(17 * list(CASES).index(case) + len(kind), batch, hkv, dp, cap, kind)
    multi = _run(_lib.TB_SELECT_MULTI_KERNEL, dm, Kp, qp, ctx, sink, window, budget, nbr, reduce)
    clus = _run(_lib.TB_SELECT_CLUSTER, dm, Kp, qp, ctx, sink, window, budget, nbr, reduce)
    for name, a, b in zip(("idx", "count", "sel_bits"), multi[:3], clus[:3]):
        assert np.array_equal(a, b), f"{name} differs between the routes"
    assert np.array_equal(multi[3], clus[3], equal_nan=True), "scores differ between the routes"
    # the sets are what they should be in size: all of C, nothing, or at least the budget
    for b in range(batch):
        nC = max(ctx[b] - window - sink, 0)
        rows = range(0, 4 * hkv, 4) if reduce is not None else range(4 * hkv)
        for h in rows:
            c = int(clus[1][b, h])
            if nC <= budget:
                assert c == nC
            else:
                assert budget <= c <= min((2 * nbr + 1) * budget, nC)


def test_forced_cluster_route_refuses_what_does_not_fit():
    # past 16 CTAs x 16 warps x 16 words x 32 positions per head row
    dm = tb.dims(batch=1, n_q_heads=4, n_kv_heads=1, head_dim=128, d_proj=32, ctx_cap=140_000)
    Kp, qp = _inputs(1, 1, 1, 32, 140_000, "normal")
    with pytest.raises(tb.TbError) as e:
        _run(_lib.TB_SELECT_CLUSTER, dm, Kp, qp, [130_000], 16, 64, 1024, 1, None)
    assert e.value.status == _lib.TB_ERR_UNSUPPORTED
    assert _lib.load().tb_select_algorithm() == _lib.TB_SELECT_AUTO
    # one score row per group: its keys take fewer registers, so longer slices fit
    multi = _run(_lib.TB_SELECT_MULTI_KERNEL, dm, Kp, qp, [130_000], 16, 64, 1024, 1, "max")
    clus = _run(_lib.TB_SELECT_CLUSTER, dm, Kp, qp, [130_000], 16, 64, 1024, 1, "max")
    for a, b in zip(multi[:3], clus[:3]):
        assert np.array_equal(a, b)


def test_graph_kernel_count_follows_the_route():
    """bench.py reports the libtb kernels its graphs launch by counting the
    graph's kernel nodes; one selection call is 3 kernels on the multi-kernel
    route and 2 (scoring, then the cluster selection) on the cluster route."""
    import bench
    batch, hkv, dp, cap, ctx, sink, window, budget, nbr = CASES["ragged_modes"]
    dm = tb.dims(batch=batch, n_q_heads=4 * hkv, n_kv_heads=hkv, head_dim=128, d_proj=dp, ctx_cap=cap)
    Kp, qp = _inputs(3, batch, hkv, dp, cap, "normal")
    hq, W = dm.n_q_heads, (cap + 31) // 32
    idx = torch.zeros((batch, hq, min((2 * nbr + 1) * budget, cap)), dtype=torch.int32, device=DEV)
    cnt = torch.zeros((batch, hq), dtype=torch.int32, device=DEV)
    bits = torch.zeros((batch, hq, W), dtype=torch.int32, device=DEV)
    ws = tb.workspace(tb.score_select_workspace_bytes(dm))
    ctx_t = torch.tensor(ctx, dtype=torch.int32, device=DEV)
    st = torch.cuda.Stream()
    counts = {}
    for algo in (_lib.TB_SELECT_MULTI_KERNEL, _lib.TB_SELECT_CLUSTER):
        _lib.select_set_algorithm(algo)
        try:
            tb.score_select(dm, qp, hq * dp, Kp, ctx_t, sink, window, budget, nbr, idx, cnt, bits, ws)  # set-up
            torch.cuda.synchronize()
            g = bench.capture(lambda s: tb.score_select(dm, qp, hq * dp, Kp, ctx_t, sink, window, budget, nbr, idx,
                                                        cnt, bits, ws, stream=s), st, count_kernels=True)
        finally:
            _lib.select_set_algorithm(_lib.TB_SELECT_AUTO)
        g.replay()
        torch.cuda.synchronize()
        counts[algo] = g.libtb_kernels
    assert counts == {_lib.TB_SELECT_MULTI_KERNEL: 3, _lib.TB_SELECT_CLUSTER: 2}


def test_cluster_route_on_a_reused_workspace():
    """The cluster route keeps each score row's key range in its workspace
    between the scoring and the selection kernel and clears it again; calls
    that reuse one workspace, with inputs of different ranges and with the
    other route in between, must each give the multi-kernel route's result."""
    batch, hkv, dp, cap, ctx, sink, window, budget, nbr = CASES["llama64k_layer"]
    dm = tb.dims(batch=batch, n_q_heads=4 * hkv, n_kv_heads=hkv, head_dim=128, d_proj=dp, ctx_cap=cap)
    hq, W = dm.n_q_heads, (cap + 31) // 32
    icap = min((2 * nbr + 1) * budget, cap)
    ws = tb.workspace(tb.score_select_workspace_bytes(dm))
    ctx_t = torch.tensor(ctx, dtype=torch.int32, device=DEV)

    def call(algo, Kp, qp):
        idx = torch.full((batch, hq, icap), -7, dtype=torch.int32, device=DEV)
        cnt = torch.full((batch, hq), -7, dtype=torch.int32, device=DEV)
        bits = torch.full((batch, hq, W), -1, dtype=torch.int32, device=DEV)
        _lib.select_set_algorithm(algo)
        try:
            tb.score_select(dm, qp, hq * dp, Kp, ctx_t, sink, window, budget, nbr, idx, cnt, bits, ws)
        finally:
            _lib.select_set_algorithm(_lib.TB_SELECT_AUTO)
        torch.cuda.synchronize()
        return idx.cpu().numpy(), cnt.cpu().numpy(), bits.cpu().numpy()

    order = [("normal", _lib.TB_SELECT_CLUSTER), ("outlier", _lib.TB_SELECT_CLUSTER),
             ("coarse", _lib.TB_SELECT_MULTI_KERNEL), ("normal", _lib.TB_SELECT_CLUSTER),
             ("coarse", _lib.TB_SELECT_CLUSTER)]
    for i, (kind, algo) in enumerate(order):
        Kp, qp = _inputs(100 + i, batch, hkv, dp, cap, kind)
        if kind == "normal":
            qp = qp * (10.0 ** (i - 2))  # another score range on each call
        got = call(algo, Kp, qp)
        fresh = _run(_lib.TB_SELECT_MULTI_KERNEL, dm, Kp, qp, ctx, sink, window, budget, nbr, None)
        for name, a, b in zip(("idx", "count", "sel_bits"), fresh[:3], got):
            assert np.array_equal(a, b), f"call {i} ({kind}): {name} differs from a fresh multi-kernel call"
    assert tb.workspace_check(ws) == 0
