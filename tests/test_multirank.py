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
