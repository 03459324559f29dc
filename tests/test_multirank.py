"""The multi-rank host logic of the benchmark on CPU with gloo (world size 2):
every rank decodes its own seeded replica, the job time is the slowest
rank's, and the reported rate counts every rank's tokens."""
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
