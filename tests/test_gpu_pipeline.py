"""The tiny integer-valued workload end to end through the CUDA path against
the oracle's own decode loop (bit-exact selection in every mode), and graph
replay of a multi-layer schedule equal to eager execution.  The multi-layer
schedule checks against the oracle are in test_gpu_schedule.py."""
import math

import numpy as np
import pytest
import torch

import oracle
import parity
import tb_inputs
from oracle import schedule as oschedule
from query_aware_sparse_tb_b200.decode import DecodeShape, SparseDecoder

pytestmark = pytest.mark.gpu
DEV = "cuda"


class HostData:
    def __init__(self, w, run):
        self.w, self.run = w, run

    def kv(self, l):
        return parity.bits16(self.run["K"][l]), parity.bits16(self.run["V"][l])

    def wk(self, l):
        return parity.bits16(self.run["Wk"][l])

    def mlp(self, p):
        W1, W2 = self.run["mlp"][p]
        return parity.bits16(W1), parity.bits16(W2)

    def h(self, k, p):
        return parity.bits16(tb_inputs.hidden_state(self.w, k, p, DEV))

    def qp_direct(self, k, l):
        return tb_inputs.direct_qp(self.w, k, l, DEV).cpu().numpy()

    def q(self, i, l):
        return parity.bits16(tb_inputs.query(self.w, i, l, DEV))


def _setup(w, selection="head"):
    K, V, Wk = [], [], []
    for l in range(w.n_layers):
        k, v = tb_inputs.kv_layer(w, l, DEV)
        K.append(k)
        V.append(v)
        Wk.append(tb_inputs.wk_layer(w, l, DEV))
    stride = w.producer_stride if w.hidden > 0 else 1
    mlp = {p: tb_inputs.mlp_weights(w, p, DEV) for p in range(0, w.n_layers, stride)} if w.hidden > 0 else {}
    shape = DecodeShape(batch=w.batch, n_layers=w.n_layers, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                        head_dim=w.head_dim, d_proj=w.d_proj, hidden=w.hidden, inter=w.inter, stride=stride,
                        sink=w.sink, window=w.window, budget=w.budget, nbr=w.nbr, interval=w.interval,
                        ctx_cap=w.ctx_cap)
    dec = SparseDecoder(shape, K, V, Wk, mlp, w.ctx0_per_seq(), w.steps, DEV, selection=selection)
    return dec, dict(K=K, V=V, Wk=Wk, mlp=mlp)


def _step_inputs(w, i):
    nL = w.n_layers
    Q = torch.stack([tb_inputs.query(w, i, l, DEV) for l in range(nL)])
    k = i // w.interval
    if w.hidden > 0:
        stride = w.producer_stride
        h = torch.stack([tb_inputs.hidden_state(w, k, p, DEV) for p in range(0, nL, stride)])
        return Q, h, None
    return Q, None, torch.stack([tb_inputs.direct_qp(w, k, l, DEV) for l in range(nL)])


@pytest.mark.parametrize("selection", ["head", "group_max", "group_sum", "inclusive"])
def test_tiny300_end_to_end_bit_exact_selection(selection):
    # integer-valued inputs: every score is exact, so the sets must match bit for bit
    w = tb_inputs.WORKLOADS["tiny300"]
    dec, run = _setup(w, selection)
    dec.prefill()
    Q, _, qd = _step_inputs(w, 0)
    out = torch.zeros(1, 1, w.n_q_heads, w.head_dim, device=DEV)
    dec.step(0, Q, out, qp_direct=qd)
    torch.cuda.synchronize()
    ref = oschedule.run(w, HostData(w, run), layers=[0], steps=1, selection=selection)[(0, 0)]
    for h in range(w.n_q_heads):
        got = dec.idx[0][0, h, :dec.cnt[0][0, h]].cpu().numpy()
        assert np.array_equal(got, ref["idx"][0][h]), h
    parity.assert_close(out[0].cpu().numpy(), ref["out"], "tiny300 out")


def _small_llama():
    return tb_inputs.WORKLOADS["llama8k"].scaled(
        name="pipe_small", n_layers=4, n_q_heads=8, n_kv_heads=2, hidden=512, inter=256, producer_stride=2,
        batch=2, ctx0=0, ctx0_lo=650, ctx0_hi=900, sink=8, window=64, budget=48, interval=4, steps=12)


def test_graph_replay_equals_eager():
    w = _small_llama().scaled(name="pipe_graph", steps=8)
    dec, _ = _setup(w)
    dec.prefill()
    inputs = [_step_inputs(w, i) for i in range(w.steps)]
    out = torch.zeros(w.n_layers, w.batch, w.n_q_heads, w.head_dim, device=DEV)
    outs_eager = []
    for i in range(w.steps):
        Q, h, qd = inputs[i]
        dec.step(i, Q, out, h=h, qp_direct=qd)
        outs_eager.append(out.clone())
    idx_eager = [t.clone() for t in dec.idx]
    snaps = [torch.zeros_like(out) for _ in range(w.steps)]
    st = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        for i in range(w.steps):
            Q, h, qd = inputs[i]
            dec.step(i, Q, out, h=h, qp_direct=qd)
            snaps[i].copy_(out)
    g.replay()
    torch.cuda.synchronize()
    for i in range(w.steps):
        assert torch.equal(snaps[i], outs_eager[i]), i
    for a, b in zip(idx_eager, dec.idx):
        assert torch.equal(a, b)
