"""The whole decode schedule through the CUDA path against the oracle's own
decode loop (tests/schedule_check.py describes every check):

  * a small multi-layer, ragged-batch shape in all four selection modes, every
    head and every step;
  * the single-layer Llama-shaped workload exactly as configured (8192-token
    context, predictor MLP 4096 -> 1024 -> 32 x 32, budget 1024, prediction
    interval 16 over 64 decode steps), every head and every step;
  * the three large workloads at full context and batch, four layers (one
    producer layer and the layers its four query slots serve), across at
    least one whole prediction interval, on sampled sequences and KV heads;
    the 64K case runs to step 64, so the prediction there reads the key batch
    projected at step 63;
  * the decoder's extra selection streams (the layers' selections round-robin
    over two or four streams) against all selections on one stream, bit for
    bit.
"""
import pytest

import bench
import schedule_check as sc
import tb_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _small():
    return tb_inputs.WORKLOADS["llama8k"].scaled(
        name="pipe_small", n_layers=4, n_q_heads=8, n_kv_heads=2, hidden=512, inter=256, producer_stride=2,
        batch=2, ctx0=0, ctx0_lo=650, ctx0_hi=900, sink=8, window=64, budget=48, interval=4, steps=12)


@pytest.mark.parametrize("selection", ["head", "group_max", "group_sum", "inclusive"])
def test_small_multi_layer_schedule(selection):
    w = _small()
    run = bench.Run(w, DEV, selection=selection)
    run.dec.prefill()
    st = sc.check_schedule(run, layers=list(range(w.n_layers)), steps=w.steps, seqs=list(range(w.batch)),
                           heads=list(range(w.n_q_heads)), attn_steps=range(w.steps), selection=selection)
    n_pred = (w.steps + w.interval - 1) // w.interval
    assert st["selections"] == n_pred * w.n_layers * w.batch * w.n_q_heads
    assert st["outputs"] >= w.steps * w.n_layers * w.batch * w.n_q_heads


def test_llama8k_as_configured():
    w = tb_inputs.WORKLOADS["llama8k"]
    run = bench.Run(w, DEV)
    run.dec.prefill()
    st = sc.check_schedule(run, layers=[0], steps=w.steps, seqs=[0], heads=list(range(w.n_q_heads)),
                           attn_steps=range(w.steps))
    assert st["selections"] == (w.steps // w.interval) * w.n_q_heads
    assert st["outputs"] >= w.steps * w.n_q_heads


@pytest.mark.parametrize("name,steps,attn_steps,seqs,groups", [
    ("llama64k", 65, [0, 1, 15, 16, 17, 63, 64], [0], [0, 7]),
    ("batch16", 17, [0, 1, 7, 8, 16], [0, 9, 15], [2, 5]),
    ("long256k", 17, [0, 1, 15, 16], [0], [0, 6]),
])
def test_full_size_multi_step(name, steps, attn_steps, seqs, groups):
    w = tb_inputs.WORKLOADS[name].scaled(n_layers=4)     # one producer layer and its 4 query slots
    assert w.producer_stride == 4
    run = bench.Run(w, DEV, steps=steps)
    run.dec.prefill()
    heads = sc.sampled_heads(w, groups)
    st = sc.check_schedule(run, layers=list(range(4)), steps=steps, seqs=seqs, heads=heads, attn_steps=attn_steps)
    n_pred = (steps + w.interval - 1) // w.interval
    assert st["selections"] == n_pred * 4 * len(seqs) * len(heads)
    assert st["outputs"] >= len(attn_steps) * 4 * len(seqs) * len(heads)


@pytest.mark.parametrize("selection,streams", [("head", 2), ("head", 4), ("group_max", 4)])
def test_overlapped_selections_equal_one_stream(selection, streams):
    """The schedule checks above pass on_select, which keeps every selection
    on one stream; here the decoder spreads the layers' selections over the
    caller's stream and one or three more (each with its own selection and plan
    workspaces), eagerly and replayed from a CUDA graph, and must
    leave every index list, count, bitmap and output of the one-stream run."""
    import torch
    w = _small()
    runs = {ov: bench.Run(w, DEV, selection=selection, overlap_select=ov, select_streams=streams)
            for ov in (False, True)}
    assert len(runs[True].dec.sel_lanes) == streams - 1 and not runs[False].dec.sel_lanes
    for r in runs.values():
        r.dec.prefill()
    torch.cuda.synchronize()
    for i in range(w.steps):
        got = {}
        for ov, r in runs.items():
            Q, h, qd = r.step_inputs(i)
            r.dec.step(i, Q, r.out, h=h, qp_direct=qd)
            torch.cuda.synchronize()
            got[ov] = [t.clone() for t in r.dec.idx + r.dec.cnt + r.dec.bits] + [r.out.clone()]
        for a, b in zip(got[False], got[True]):
            assert torch.equal(a, b), f"step {i}: the overlapped selections differ from one stream"
    for r in runs.values():
        for ws in r.dec.workspaces():
            assert bench.L.workspace_check(ws) == 0
    # the same steps captured in one graph (fork and join inside the capture)
    r = runs[True]
    ref = runs[False]
    st = torch.cuda.Stream()
    for i in range(w.steps):
        Q, h, qd = r.step_inputs(i)
        g = bench.capture(lambda s, i=i, Q=Q, h=h, qd=qd: r.dec.step(i, Q, r.out, h=h, qp_direct=qd, stream=s), st)
        g.replay()
        torch.cuda.synchronize()
        Qr, hr, qdr = ref.step_inputs(i)
        ref.dec.step(i, Qr, ref.out, h=hr, qp_direct=qdr)
        torch.cuda.synchronize()
        for a, b in zip(r.dec.idx + r.dec.cnt + r.dec.bits + [r.out], ref.dec.idx + ref.dec.cnt + ref.dec.bits + [ref.out]):
            assert torch.equal(a, b), f"step {i}: the graph-replayed overlapped step differs"
