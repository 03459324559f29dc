"""The K/V prefetch launch mode against its contract: every decode step first
appends the token's K and V rows with tb_kv_append (on steps with neither a
projection nor a prediction that append is the kernel right before the first
attention launch, which may read every row below T-1 before the append has
finished).  Row T-1 must still be read after it lands: the decode loop starts
from caches whose decode rows are zero and must reproduce the oracle's
schedule over the full caches."""
import pytest
import torch

import bench
import parity
import schedule_check as sc
import tb_inputs
import query_aware_sparse_tb_b200 as tb

pytestmark = pytest.mark.gpu
DEV = "cuda"


class FullData(sc.RunData):
    """The oracle's view: the caches as they are once every row is appended."""

    def __init__(self, run, K, V):
        super().__init__(run)
        self.K, self.V = K, V

    def kv(self, l):
        return parity.bits16(self.K[l]), parity.bits16(self.V[l])


@pytest.mark.parametrize("hidden", [0, 512])
def test_prefetch_reads_the_row_the_preceding_append_writes(hidden):
    w = tb_inputs.WORKLOADS["llama8k"].scaled(
        name="prefetch_append", n_layers=3, n_q_heads=8, n_kv_heads=2, hidden=hidden, inter=256 if hidden else 0,
        producer_stride=3 if hidden else 1, batch=2, ctx0=0, ctx0_lo=700, ctx0_hi=900, sink=8, window=64,
        budget=48, interval=4, steps=70)
    run = bench.Run(w, DEV)
    assert run.dec.prefetch_kv
    full_K = [k.clone() for k in run.K]
    full_V = [v.clone() for v in run.V]
    ctx0 = run.ctx0
    for l in range(w.n_layers):
        for b in range(w.batch):
            run.K[l][b, :, ctx0[b]:] = 0
            run.V[l][b, :, ctx0[b]:] = 0
    run.dec.prefill()
    caches = torch.tensor([p for l in range(w.n_layers) for p in (run.K[l].data_ptr(), run.V[l].data_ptr())],
                          dtype=torch.int64, device=DEV)
    src = torch.empty(w.n_layers, 2, w.batch, w.n_kv_heads, w.head_dim, dtype=torch.bfloat16, device=DEV)
    ws = tb.workspace(256)

    def append(i):
        for l in range(w.n_layers):
            for b in range(w.batch):
                src[l, 0, b] = full_K[l][b, :, ctx0[b] + i]
                src[l, 1, b] = full_V[l][b, :, ctx0[b] + i]
        tb.kv_append(run.dec.dims, w.n_layers, src, caches, run.dec.ctx[i], ws)

    st = sc.check_schedule(run, layers=list(range(w.n_layers)), steps=w.steps, seqs=list(range(w.batch)),
                           heads=list(range(w.n_q_heads)), attn_steps=range(w.steps),
                           data=FullData(run, full_K, full_V), before_step=append)
    assert tb.workspace_check(ws) == 0
    assert st["outputs"] >= w.steps * w.n_layers * w.batch * w.n_q_heads
    for l in range(w.n_layers):                          # the caches now hold every appended row
        for b in range(w.batch):
            e = ctx0[b] + w.steps
            assert torch.equal(run.K[l][b, :, :e], full_K[l][b, :, :e])
