"""The end-to-end measurement's loop (bench.E2E), as the bench records it in
a CUDA graph: inputs copied from pinned host memory and outputs copied back
on a copy stream, double buffered, overlapping the next step's compute.  Its
host-side outputs must be the device-resident loop's outputs, bit for bit:
any slot reused too early would show."""
import pytest
import torch

import bench
import tb_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("hidden", [0, 512])
def test_e2e_loop_returns_the_device_resident_outputs(hidden):
    w = tb_inputs.WORKLOADS["llama8k"].scaled(
        name="e2e_overlap", n_layers=3, n_q_heads=8, n_kv_heads=2, hidden=hidden, inter=256 if hidden else 0,
        producer_stride=3 if hidden else 1, batch=2, ctx0=0, ctx0_lo=700, ctx0_hi=900, sink=8, window=64,
        budget=48, interval=4, steps=40)
    run = bench.Run(w, "cuda")
    run.dec.prefill()
    torch.cuda.synchronize()
    e2e = bench.E2E(run)
    st = torch.cuda.Stream()
    g = bench.capture(e2e.body, st)
    for _ in range(2):  # a replay starts where the last one left the buffers
        g.replay()
    torch.cuda.synchronize()
    host_out = e2e.out_host.clone()
    for i in range(run.steps):
        Q, h, qd = run.step_inputs(i)
        run.dec.step(i, Q, run.out, h=h, qp_direct=qd)
        torch.cuda.synchronize()
        assert torch.equal(run.out.cpu(), host_out[i]), f"step {i}: the e2e loop's outputs differ"
