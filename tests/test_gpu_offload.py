"""The CPU-offloaded KV cache (TokenButler summaries, "Contributions": CPU
offloading; "Results": per-token latency at 256K+ tokens): K and V live in
pinned host memory that the attention kernels read directly, K' and the
selection stay on the device, and each batch of new keys is projected from a
device staging copy.  The offloaded run must reproduce the device-resident
run bit for bit (the same kernels on the same bytes, in the same order), and
the whole offloaded schedule must pass the schedule checks against the
oracle's own decode loop (every head, every step)."""
import numpy as np
import pytest
import torch

import bench
import parity
import schedule_check as sc
import tb_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _small():
    return tb_inputs.WORKLOADS["llama8k"].scaled(
        name="offload_small", n_layers=2, n_q_heads=8, n_kv_heads=2, hidden=512, inter=256, producer_stride=2,
        batch=2, ctx0=0, ctx0_lo=650, ctx0_hi=900, sink=8, window=64, budget=48, interval=4, steps=40)


def test_offloaded_run_equals_device_run():
    w = _small()
    dev = bench.Run(w, DEV)
    off = bench.Run(w, DEV, offload=True)
    K_ref = [parity.bits16(k) for k in dev.K]
    V_ref = [parity.bits16(v) for v in dev.V]
    for run in (dev, off):
        run.dec.prefill()
    off.dec.offload()
    off.K = off.V = None
    assert off.dec.proj_steps, "the schedule must include projection batches during decoding"
    for i in range(w.steps):
        outs = []
        for run in (dev, off):
            Q, h, qd = run.step_inputs(i)
            run.dec.step(i, Q, run.out, h=h, qp_direct=qd)
            outs.append(run.out.clone())
        dense = []
        for run in (dev, off):
            out = torch.empty_like(run.out[0])
            run.dec.attend_dense(i, 1, run.Q[i][1], out)
            dense.append(out)
        torch.cuda.synchronize()
        assert torch.equal(outs[0], outs[1]), f"sparse outputs differ at step {i}"
        assert torch.equal(dense[0], dense[1]), f"dense outputs differ at step {i}"
        for l in range(w.n_layers):
            assert torch.equal(dev.dec.Kp[l], off.dec.Kp[l]), (i, l)
            assert torch.equal(dev.dec.idx[l], off.dec.idx[l]), (i, l)
    for ws in (off.dec.ws_attn, off.dec.ws_sel, off.dec.ws_proj, off.dec.ws_pred):
        assert bench.L.workspace_check(ws) == 0
    # the host copies hold the cache the device run attends to
    assert np.array_equal(parity.bits16(off.dec.K_host[0].tensor), K_ref[0])
    for hb in off.dec.K_host + off.dec.V_host:
        hb.free()


def test_offloaded_schedule_against_oracle():
    w = _small().scaled(steps=20)
    run = bench.Run(w, DEV, offload=True)
    run.dec.prefill()
    run.dec.offload()
    run.K = run.V = None
    st = sc.check_schedule(run, layers=list(range(w.n_layers)), steps=w.steps, seqs=list(range(w.batch)),
                           heads=list(range(w.n_q_heads)), attn_steps=range(w.steps))
    assert st["outputs"] >= w.steps * w.n_layers * w.batch * w.n_q_heads
    for hb in run.dec.K_host + run.dec.V_host:
        hb.free()
