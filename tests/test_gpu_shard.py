"""KV-head sharding on one GPU: the ranks' shares of a workload (each rank's
KV heads, their query heads and the predictor rows that emit their queries),
run one after another through the unchanged entry points, reproduce the
unsharded run.  Projected keys, predicted queries and selected sets are
bit-identical (every per-head computation is the same arithmetic); attention
outputs agree within the attention tolerance (the split count over the
context depends on how many (sequence, KV head) pairs a launch holds).  The
ranks never wait on one another, so running them in sequence on one GPU is
exactly what separate GPUs would compute."""
import pytest
import torch

import bench
import parity
import tb_inputs
from query_aware_sparse_tb_b200.decode import gather_head_outputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("world", [2])
def test_kv_head_shards_reproduce_the_unsharded_run(world):
    w = tb_inputs.WORKLOADS["llama8k"].scaled(
        name="shard_small", n_layers=4, n_q_heads=8, n_kv_heads=2, hidden=512, inter=256, producer_stride=2,
        batch=2, ctx0=0, ctx0_lo=650, ctx0_hi=900, sink=8, window=64, budget=48, interval=4, steps=9)
    full = bench.Run(w, DEV)
    shards = [bench.Run(w, DEV, shard=(r, world)) for r in range(world)]
    for run in [full] + shards:
        run.dec.prefill()
    heads = [r.q_heads for r in shards]
    for i in range(w.steps):
        outs = []
        for run in [full] + shards:
            Q, h, qd = run.step_inputs(i)
            run.dec.step(i, Q, run.out, h=h, qp_direct=qd)
            outs.append(run.out.clone())
        torch.cuda.synchronize()
        got = gather_head_outputs(outs[1:], heads)
        parity.assert_close(got.cpu().numpy(), outs[0].cpu().numpy(), f"step {i}")
        for l in range(w.n_layers):
            for run in shards:
                g0, g1 = run.kv_heads.start, run.kv_heads.stop
                h0, h1 = run.q_heads.start, run.q_heads.stop
                assert torch.equal(run.dec.Kp[l], full.dec.Kp[l][:, g0:g1]), (i, l)
                assert torch.equal(run.dec.idx[l], full.dec.idx[l][:, h0:h1]), (i, l)
                assert torch.equal(run.dec.cnt[l], full.dec.cnt[l][:, h0:h1]), (i, l)
                assert torch.equal(run.dec.bits[l], full.dec.bits[l][:, h0:h1]), (i, l)
        for p in full.producers:
            for run in shards:
                h0, h1 = run.q_heads.start, run.q_heads.stop
                assert torch.equal(run.dec.qp[p], full.dec.qp[p][:, :, h0:h1]), (i, p)
    for run in [full] + shards:
        for ws in (run.dec.ws_attn, run.dec.ws_sel, run.dec.ws_proj, run.dec.ws_pred):
            assert bench.L.workspace_check(ws) == 0
