"""The multi-rank host logic on CPU with gloo (world sizes 2 and 3): every
rank decodes its own seeded replica, the job time is the slowest rank's, and
the reported rate counts every rank's tokens; KV-head sharding and context
sharding reproduce the single-device oracle results from the ranks' shares
and their exchanges."""
import math
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import tb_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, "cpu")
        w = bench.replica(tb_inputs.WORKLOADS["tiny300"], rank)
        K, _ = tb_inputs.kv_layer(w, 0, "cpu")
        digest = float(K.float().abs().sum())
        gathered = [None] * world
        dist.all_gather_object(gathered, (w.seed, digest))
        q.put((rank, ms, gathered))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, gathered in results:
        assert ms == 15.0, "every rank sees the slowest rank's time"
        seeds = [g[0] for g in gathered]
        digests = [g[1] for g in gathered]
        assert seeds == [0, 1], "each rank has its own replica seed"
        assert digests[0] != digests[1], "replicas hold different data"


def test_rate_helpers_single_process():
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.aggregate_rate(1, 256, 500.0) == pytest.approx(512.0)
    assert bench.aggregate_rate(8, 256, 500.0) == pytest.approx(4096.0)
    w = bench.replica(tb_inputs.WORKLOADS["llama64k"], 3)
    assert w.seed == 3 and w.ctx0 == 65536


# ------------------------------------------------------------ KV-head sharding

def _local_outputs(w, qh, kvh):
    """One rank's share of a decode step of the tiny workload, computed by the
    oracle on the rank's slices of the inputs: K, V, W_k of its KV heads, Q and
    q' of their query heads."""
    import math

    import numpy as np

    import oracle
    import parity
    K, V = tb_inputs.kv_layer(w, 0, "cpu")
    Kl, Vl = parity.bits16(K[:, kvh.start:kvh.stop]), parity.bits16(V[:, kvh.start:kvh.stop])
    Wk = parity.bits16(tb_inputs.wk_layer(w, 0, "cpu")[kvh.start:kvh.stop])
    Q = parity.bits16(tb_inputs.query(w, 0, 0, "cpu")[:, qh.start:qh.stop])
    qp = tb_inputs.direct_qp(w, 0, 0, "cpu")[:, qh.start:qh.stop].numpy()
    T = w.ctx0 + 1
    out = np.zeros((w.batch, len(qh), w.head_dim), np.float32)
    for j in range(len(qh)):
        g = j // w.group                                   # local KV head of local query head j
        Kp = oracle.project_keys(Kl[0, g, :T], Wk[g])
        s = oracle.scores(qp[0, j], Kp, w.sink, T - w.window)
        I = oracle.select(s, T, w.sink, w.window, w.budget, w.nbr)
        A = oracle.attention_set(T, w.sink, w.window, I)
        out[0, j] = oracle.attention(Q[0, j], Kl[0, g], Vl[0, g], A, 1 / math.sqrt(w.head_dim))
    return out


def _shard_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from query_aware_sparse_tb_b200.decode import gather_head_outputs, kv_head_shard
        w = tb_inputs.WORKLOADS["tiny300"]
        kvh, qh = kv_head_shard(w.n_kv_heads, w.group, rank, world)
        local = torch.from_numpy(_local_outputs(w, qh, kvh))
        parts = [torch.empty_like(local) for _ in range(world)]
        dist.all_gather(parts, local)
        full = gather_head_outputs(parts, [kv_head_shard(w.n_kv_heads, w.group, r, world)[1] for r in range(world)])
        q.put((rank, full.numpy()))
    finally:
        dist.destroy_process_group()


def test_kv_head_sharding_two_ranks_gloo():
    # two ranks each own one KV head of the tiny workload and its 4 query
    # heads; their gathered outputs equal the unsharded oracle run exactly
    import numpy as np

    import parity
    from oracle import schedule as oschedule
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = tb_inputs.WORKLOADS["tiny300"]

    class Data:
        def kv(self, l):
            K, V = tb_inputs.kv_layer(w, l, "cpu")
            return parity.bits16(K), parity.bits16(V)

        def wk(self, l):
            return parity.bits16(tb_inputs.wk_layer(w, l, "cpu"))

        def qp_direct(self, k, l):
            return tb_inputs.direct_qp(w, k, l, "cpu").numpy()

        def q(self, i, l):
            return parity.bits16(tb_inputs.query(w, i, l, "cpu"))

    ref = oschedule.run(w, Data(), layers=[0], steps=1)[(0, 0)]["out"]
    for rank, full in results:
        assert np.array_equal(full, ref), f"rank {rank}: gathered outputs differ from the unsharded run"


def test_kv_head_shard_assignment():
    from query_aware_sparse_tb_b200.decode import kv_head_shard
    for world in (1, 2, 4, 8):
        owned = [kv_head_shard(8, 4, r, world) for r in range(world)]
        assert sorted(g for kvh, _ in owned for g in kvh) == list(range(8))
        assert sorted(h for _, qh in owned for h in qh) == list(range(32))
        for kvh, qh in owned:
            assert list(qh) == [h for g in kvh for h in range(4 * g, 4 * g + 4)]
    with pytest.raises(ValueError):
        kv_head_shard(8, 4, 0, 3)


def test_sharded_predictor_rows_give_the_sharded_queries():
    # the second matrix's rows of a rank's heads, in every slot, give exactly
    # that rank's slice of the unsharded predictor output (oracle, exact)
    import numpy as np

    import oracle
    import parity
    from query_aware_sparse_tb_b200.decode import kv_head_shard, shard_w2
    w = tb_inputs.WORKLOADS["llama64k"].scaled(name="shard_mlp", hidden=256, inter=256, n_q_heads=8, n_kv_heads=2,
                                                batch=3)
    W1, W2 = tb_inputs.mlp_weights(w, 0, "cpu")
    h = tb_inputs.hidden_state(w, 0, 0, "cpu")
    full = oracle.predict_queries(parity.bits16(h), parity.bits16(W1), parity.bits16(W2)).reshape(
        w.batch, w.slots, w.n_q_heads, w.d_proj)
    for rank in range(2):
        _, qh = kv_head_shard(w.n_kv_heads, w.group, rank, 2)
        W2r = shard_w2(W2, w.slots, w.n_q_heads, w.d_proj, qh)
        assert W2r.shape == (w.slots * len(qh) * w.d_proj, w.inter)
        got = oracle.predict_queries(parity.bits16(h), parity.bits16(W1), parity.bits16(W2r)).reshape(
            w.batch, w.slots, len(qh), w.d_proj)
        assert np.array_equal(got, full[:, :, qh.start:qh.stop])


# ------------------------------------------------------------ context sharding

def _cp_case():
    return tb_inputs.WORKLOADS["tiny300"].scaled(name="cp_tiny", ctx0=700, ctx0_lo=700, ctx0_hi=700, budget=40)


def _cp_worker(rank, world, port, q):
    # one rank's share of a context-sharded step, computed by the oracle on the
    # rank's block: its local top-B, the exchange of candidates, the merge and
    # its block's part of the attention as an unnormalised (m, l, o) state
    import numpy as np

    import oracle
    import parity
    from query_aware_sparse_tb_b200.decode import context_blocks, local_rows, local_selection_params
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = _cp_case()
        T = w.ctx0 + 1
        blk = context_blocks(w.ctx_cap, world, w.window)[rank]
        K, V = tb_inputs.kv_layer(w, 0, "cpu")
        Kb, Vb = parity.bits16(K), parity.bits16(V)
        Wk = parity.bits16(tb_inputs.wk_layer(w, 0, "cpu"))
        qp = tb_inputs.direct_qp(w, 0, 0, "cpu").numpy()
        Q = parity.bits16(tb_inputs.query(w, 0, 0, "cpu"))
        lT, lS = local_selection_params(T, blk, w.sink, w.window)
        rows = local_rows(T, blk)
        cands = {}
        for h in range(w.n_q_heads):
            g = h // w.group
            Kp = oracle.project_keys(Kb[0, g, blk[0]:blk[0] + max(0, lT - w.window)], Wk[g])
            s = oracle.scores(qp[0, h], Kp, lS, lT - w.window) if lT - w.window > lS else np.zeros(0, np.float32)
            top = oracle.select(s, lT, lS, w.window, w.budget, 0)
            cands[h] = [(float(s[t - lS]), int(t + blk[0])) for t in top]
        allc = [None] * world
        dist.all_gather_object(allc, cands)
        parts = {}
        for h in range(w.n_q_heads):
            pool = sorted((c for rc in allc for c in rc[h]), key=lambda c: (-c[0], c[1]))[:w.budget]
            lo, hi = w.sink, T - w.window
            I = sorted({t + k for _, t in pool for k in range(-w.nbr, w.nbr + 1) if lo <= t + k < hi})
            A = [t for t in oracle.attention_set(T, w.sink, w.window, np.array(I, np.int32))
                 if blk[0] <= t < blk[0] + rows and t < T]
            g = h // w.group
            qv = parity.bf16_to_f64(Q[0, h])
            if A:
                kk = parity.bf16_to_f64(Kb[0, g, A])
                vv = parity.bf16_to_f64(Vb[0, g, A])
                logit = kk @ qv / math.sqrt(w.head_dim)
                m = logit.max()
                p = np.exp(logit - m)
                parts[h] = (m, p.sum(), p @ vv, I)
            else:
                parts[h] = (-np.inf, 0.0, np.zeros(w.head_dim), I)
        allp = [None] * world
        dist.all_gather_object(allp, parts)
        q.put((rank, allp))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_sharding_gloo(world):
    # each rank holds one block of the context; the merged selection equals the
    # single-device oracle selection exactly and the combined attention equals
    # the single-device oracle attention
    import numpy as np

    import oracle
    import parity
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = _cp_case()
    T = w.ctx0 + 1
    K, V = tb_inputs.kv_layer(w, 0, "cpu")
    Kb, Vb = parity.bits16(K), parity.bits16(V)
    Wk = parity.bits16(tb_inputs.wk_layer(w, 0, "cpu"))
    qp = tb_inputs.direct_qp(w, 0, 0, "cpu").numpy()
    Q = parity.bits16(tb_inputs.query(w, 0, 0, "cpu"))
    for rank, allp in results:
        for h in range(w.n_q_heads):
            g = h // w.group
            Kp = oracle.project_keys(Kb[0, g, :T], Wk[g])
            I_ref = oracle.select(oracle.scores(qp[0, h], Kp, w.sink, T - w.window), T, w.sink, w.window, w.budget,
                                  w.nbr)
            states = [p[h] for p in allp]
            for st in states:
                assert np.array_equal(np.array(st[3], np.int64), I_ref), (rank, h)
            M = max(st[0] for st in states)
            num = sum(np.exp(st[0] - M) * st[2] for st in states if st[0] != -np.inf)
            den = sum(np.exp(st[0] - M) * st[1] for st in states if st[0] != -np.inf)
            ref = oracle.attention(Q[0, h], Kb[0, g], Vb[0, g], oracle.attention_set(T, w.sink, w.window, I_ref),
                                   1 / math.sqrt(w.head_dim))
            assert np.allclose(num / den, ref, atol=1e-6, rtol=0), (rank, h)


def test_context_block_helpers():
    from query_aware_sparse_tb_b200.decode import (block_capacity, context_blocks, local_rows,
                                                   local_selection_params)
    for cap, world, N in ((65792, 4, 64), (832, 3, 16), (300, 2, 16)):
        blocks = context_blocks(cap, world, N)
        assert blocks[0][0] == 0 and blocks[-1][1] == cap
        for (a0, a1), (b0, b1) in zip(blocks, blocks[1:]):
            assert a1 == b0 and a0 % 32 == 0 and a0 % N == 0
        for T in (1, 17, cap // 2, cap):
            covered = []
            for blk in blocks:
                lT, lS = local_selection_params(T, blk, 4, N)
                assert 1 <= lT <= block_capacity(blk, N)
                covered += [t + blk[0] for t in range(lS, lT - N)]   # the block's local candidates
                assert 1 <= local_rows(T, blk) <= blk[1] - blk[0] or blk[1] == blk[0]
            assert covered == list(range(4, max(4, T - N))), (cap, world, T)
