#!/usr/bin/env python
"""Benchmark of the TokenButler sparse decode path on B200.

One bench step = one full decode run of the workload (llama64k: 32 layers,
64K context, 256 decode steps with a prediction every 16 steps, producer every
4 layers, key projection every 64 tokens), replayed as one CUDA graph on
inputs already resident in HBM.  The same run is timed for the dense decode
kernel (the comparator) and end to end (per-step host->device copies of the
step's queries, new K/V rows and producer hidden states, and a device->host
copy of the step's outputs, all inside the graph).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference      # the CPU oracle on a bounded sample

Under torchrun every rank decodes its own independent replica (its own seeded
sequences): weak scaling, no collective on the data path; the barrier and the
max-over-ranks reduction of the device time use NCCL.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import tb_inputs  # noqa: E402
from query_aware_sparse_tb_b200 import _lib as L  # noqa: E402
from query_aware_sparse_tb_b200.decode import (DecodeShape, OffloadDecoder, SparseDecoder,  # noqa: E402
                                              is_prediction_step, kv_head_shard, record_event, shard_w2)

HBM_NOMINAL_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
ROW_BYTES_PER_DIM = 2 * 2      # K and V, bf16


# ----------------------------------------------------------------------------
# workload on the device
# ----------------------------------------------------------------------------

class Run:
    """All device buffers of one workload replica plus its decoder.  With
    shard=(rank, world) the run holds only the KV heads (and their query heads)
    that rank owns under KV-head sharding, sliced from the same seeded data."""

    def __init__(self, w: tb_inputs.Workload, device: str, steps: int | None = None, selection: str = "head",
                 shard: tuple[int, int] | None = None, offload: bool = False, balance: bool = True,
                 overlap_select: bool = True, select_streams: int = 4):
        self.w = w
        self.device = device
        self.steps = steps or w.steps
        self.ctx0 = w.ctx0_per_seq()
        nL = w.n_layers
        if shard is None:
            kvh, qh = range(w.n_kv_heads), range(w.n_q_heads)
        else:
            kvh, qh = kv_head_shard(w.n_kv_heads, w.group, *shard)
        self.kv_heads, self.q_heads = kvh, qh
        self.Hkv, self.Hq = len(kvh), len(qh)
        gs, hs = slice(kvh.start, kvh.stop), slice(qh.start, qh.stop)
        self.K, self.V, self.Wk = [], [], []
        for l in range(nL):
            K, V = tb_inputs.kv_layer(w, l, device)
            self.K.append(K[:, gs].contiguous() if shard else K)
            self.V.append(V[:, gs].contiguous() if shard else V)
            self.Wk.append(tb_inputs.wk_layer(w, l, device)[gs].contiguous())
            del K, V
        stride = w.producer_stride if w.hidden > 0 else 1
        self.producers = [l for l in range(nL) if l % stride == 0]
        self.mlp = {}
        if w.hidden > 0:
            for p in self.producers:
                W1, W2 = tb_inputs.mlp_weights(w, p, device)
                self.mlp[p] = (W1, shard_w2(W2, w.slots, w.n_q_heads, w.d_proj, qh) if shard else W2)
        self.Q = torch.stack([torch.stack([tb_inputs.query(w, i, l, device)[:, hs] for l in range(nL)])
                              for i in range(self.steps)]).contiguous()          # [steps][L][B][Hq][d]
        self.n_pred = (self.steps + w.interval - 1) // w.interval
        if w.hidden > 0:
            self.h = torch.stack([torch.stack([tb_inputs.hidden_state(w, k, p, device) for p in self.producers])
                                  for k in range(self.n_pred)])                   # [npred][nprod][B][hidden]
            self.qp_direct = None
        else:
            self.h = None
            self.qp_direct = torch.stack([torch.stack([tb_inputs.direct_qp(w, k, l, device)[:, hs]
                                                       for l in range(nL)])
                                          for k in range(self.n_pred)]).contiguous()  # [npred][L][B][Hq][d']
        self.shape = DecodeShape(batch=w.batch, n_layers=nL, n_q_heads=self.Hq, n_kv_heads=self.Hkv,
                                 head_dim=w.head_dim, d_proj=w.d_proj, hidden=w.hidden, inter=w.inter,
                                 stride=stride, sink=w.sink, window=w.window, budget=w.budget, nbr=w.nbr,
                                 interval=w.interval, ctx_cap=w.ctx_cap)
        cls = OffloadDecoder if offload else SparseDecoder
        # the bench's streams run only libtb's kernels, the K/V append of the
        # e2e loop and copies, so every attention launch may prefetch its rows
        self.dec = cls(self.shape, list(self.K), list(self.V), self.Wk, self.mlp, self.ctx0, self.steps, device,
                       selection=selection, prefetch_kv=True, balance=balance, overlap_select=overlap_select,
                       select_streams=select_streams)
        self.out = torch.zeros(nL, w.batch, self.Hq, w.head_dim, dtype=torch.float32, device=device)

    def step_inputs(self, i):
        k = i // self.w.interval
        h = self.h[k] if self.h is not None else None
        qd = self.qp_direct[k] if self.qp_direct is not None else None
        return self.Q[i], h, qd

    def run_sparse(self, stream=None, marks=None):
        for i in range(self.steps):
            Q, h, qd = self.step_inputs(i)
            self.dec.step(i, Q, self.out, h=h, qp_direct=qd, stream=stream,
                          marks=(lambda name, i=i: marks(name, i)) if marks else None)

    def run_dense(self, stream=None, marks=None):
        for i in range(self.steps):
            self.dec.dense_step(i, self.Q[i], self.out, stream=stream,
                                marks=(lambda name, i=i: marks(name, i)) if marks else None)

    # ------------------------------------------------------------ accounting
    def union_rows(self):
        """Kept (b, kv-head, t) rows of every sparse attention launch of one run,
        counting a row once for the 4 query heads of its group: sink + window +
        |OR of the group's selected bits|.  Runs the schedule once, eagerly."""
        w, dec = self.w, self.dec
        lut = torch.tensor([bin(x).count("1") for x in range(256)], dtype=torch.int64, device=self.device)
        rows = torch.zeros(self.steps, w.n_layers, dtype=torch.int64)
        sel_sizes = torch.zeros(self.steps, w.n_layers, dtype=torch.int64)
        cand = torch.zeros(self.steps, dtype=torch.int64)
        union = None
        isets = None
        for i in range(self.steps):
            Q, h, qd = self.step_inputs(i)
            dec.step(i, Q, self.out, h=h, qp_direct=qd)
            if is_prediction_step(i, w.interval):
                u = []
                s_ = []
                for l in range(w.n_layers):
                    b = dec.bits[l].view(w.batch, self.Hkv, w.group, -1)
                    orb = b[:, :, 0] | b[:, :, 1] | b[:, :, 2] | b[:, :, 3]
                    u.append(lut[orb.contiguous().view(torch.uint8).long()].sum())
                    s_.append(dec.cnt[l].sum())
                union = torch.stack(u).cpu()
                isets = torch.stack(s_).cpu()
            T = [t + i + 1 for t in self.ctx0]
            keep = sum(min(w.sink, t) + (t - max(w.sink, t - w.window)) for t in T) * self.Hkv
            rows[i] = union + keep
            sel_sizes[i] = isets
            cand[i] = sum(max(0, t - w.window - w.sink) for t in T)
        torch.cuda.synchronize()
        return rows, sel_sizes, cand

    def bytes_model(self):
        """Algorithmic HBM bytes of one run (the sum over decode steps of the
        per-step formula): sparse path, its attention part, dense path."""
        w = self.w
        d, dp = w.head_dim, w.d_proj
        rows, sel_sizes, cand = self.union_rows()
        attn_rows = rows.sum().item()
        row_b = d * ROW_BYTES_PER_DIM
        qo = self.steps * w.n_layers * w.batch * self.Hq * d * (2 + 4)
        attn_bytes = attn_rows * row_b
        sel_bytes = 0
        for i in range(self.steps):
            if is_prediction_step(i, w.interval):
                sel_bytes += w.n_layers * (self.Hkv * cand[i].item() * dp * 2)
                sel_bytes += 4 * sel_sizes[i].sum().item()
        mlp_bytes = 0
        if w.hidden > 0:
            n_out = w.slots * self.Hq * w.d_proj
            mlp_bytes = self.n_pred * len(self.producers) * (w.inter * w.hidden + n_out * w.inter) * 2
        proj_bytes = len(self.dec.proj_steps) * w.n_layers * w.batch * w.window * self.Hkv * (d + dp) * 2
        sparse_total = attn_bytes + qo + sel_bytes + mlp_bytes + proj_bytes
        dense_rows = sum(sum(t + i + 1 for t in self.ctx0) for i in range(self.steps)) * self.Hkv * w.n_layers
        dense_total = dense_rows * row_b + qo
        return dict(attn_bytes=attn_bytes, attn_rows=attn_rows, sparse_total=sparse_total, dense_total=dense_total,
                    dense_rows=dense_rows, sel_bytes=sel_bytes, mlp_bytes=mlp_bytes, proj_bytes=proj_bytes,
                    sum_head_rows=int(sel_sizes.sum().item()))


# ----------------------------------------------------------------------------
# graphs and timing
# ----------------------------------------------------------------------------

class Marks:
    """External event records at the attention-block boundaries of each
    decode step (inside a capture they are graph nodes)."""

    def __init__(self, steps):
        self.ev = {(n, i): torch.cuda.Event(enable_timing=True) for i in range(steps)
                   for n in ("attn_begin", "attn_end")}
        for ev in self.ev.values():     # torch creates the CUDA event on first record
            ev.record()
        torch.cuda.synchronize()
        self.stream = None

    def __call__(self, name, i):
        record_event(self.ev[(name, i)], self.stream)

    def attn_ms(self, steps):
        return [self.ev[("attn_begin", i)].elapsed_time(self.ev[("attn_end", i)]) for i in range(steps)]


class _KernelNodeParams(ctypes.Structure):
    _fields_ = [("func", ctypes.c_void_p), ("grid", ctypes.c_uint * 3), ("block", ctypes.c_uint * 3),
                ("shared_mem_bytes", ctypes.c_uint), ("kernel_params", ctypes.c_void_p), ("extra", ctypes.c_void_p)]


def libtb_kernel_nodes(graph) -> int:
    """Kernel nodes of a captured cudaGraph_t whose function is one of libtb's
    (C++ namespace tb): the launches one replay makes."""
    rt = ctypes.CDLL("libcudart.so.12")
    P = ctypes.c_void_p
    rt.cudaGraphGetNodes.argtypes = [P, P, ctypes.POINTER(ctypes.c_size_t)]
    rt.cudaGraphNodeGetType.argtypes = [P, ctypes.POINTER(ctypes.c_int)]
    rt.cudaGraphKernelNodeGetParams.argtypes = [P, ctypes.POINTER(_KernelNodeParams)]
    rt.cudaFuncGetName.argtypes = [ctypes.POINTER(ctypes.c_char_p), P]
    n = ctypes.c_size_t(0)
    if rt.cudaGraphGetNodes(P(graph), None, ctypes.byref(n)) != 0:
        raise RuntimeError("cudaGraphGetNodes failed")
    nodes = (P * n.value)()
    if rt.cudaGraphGetNodes(P(graph), nodes, ctypes.byref(n)) != 0:
        raise RuntimeError("cudaGraphGetNodes failed")
    count = 0
    for node in nodes:
        t = ctypes.c_int(-1)
        if rt.cudaGraphNodeGetType(P(node), ctypes.byref(t)) != 0 or t.value != 0:  # 0: kernel node
            continue
        prm = _KernelNodeParams()
        name = ctypes.c_char_p()
        if rt.cudaGraphKernelNodeGetParams(P(node), ctypes.byref(prm)) == 0 and \
                rt.cudaFuncGetName(ctypes.byref(name), prm.func) == 0 and name.value and b"_ZN2tb" in name.value:
            count += 1
    return count


def capture(fn, stream, count_kernels=False):
    """Record fn(stream) into a CUDA graph; with count_kernels the graph also
    carries `libtb_kernels`, the number of libtb kernels one replay launches."""
    g = torch.cuda.CUDAGraph(keep_graph=count_kernels)
    with torch.cuda.graph(g, stream=stream):
        fn(stream)
    if count_kernels:
        g.libtb_kernels = libtb_kernel_nodes(g.raw_cuda_graph())
        g.instantiate()
    return g


class E2E:
    """Per-step host<->device traffic of the public-API loop.  Every step, one
    host->device copy brings the step's inputs from pinned memory (all layers'
    queries and the new token's K and V rows, packed), tb_kv_append writes the
    rows into every layer's cache in one launch, prediction steps also copy the
    producer hidden states, and one device->host copy returns all layers'
    attention outputs.  The copies run on a stream of their own, double
    buffered, as a serving loop would issue them: step i+1's inputs come in
    and step i's outputs go out while step i+1 computes."""

    def __init__(self, run: Run):
        self.run = run
        w = run.w
        nL = w.n_layers
        pos = [[t + i for t in run.ctx0] for i in range(run.steps)]     # new token position T-1
        q_el = run.Q[0].numel()
        kv_el = nL * 2 * w.batch * run.Hkv * w.head_dim
        packed = torch.empty(run.steps, q_el + kv_el, dtype=torch.bfloat16)
        for i in range(run.steps):
            packed[i, :q_el] = run.Q[i].reshape(-1).cpu()
            kv = torch.empty(nL, 2, w.batch, run.Hkv, w.head_dim, dtype=torch.bfloat16)
            for l in range(nL):
                for b in range(w.batch):
                    kv[l, 0, b] = run.K[l][b, :, pos[i][b]].cpu()
                    kv[l, 1, b] = run.V[l][b, :, pos[i][b]].cpu()
            packed[i, q_el:] = kv.reshape(-1)
        self.host = packed.pin_memory()
        self.dev = [torch.empty(q_el + kv_el, dtype=torch.bfloat16, device=run.device) for _ in range(2)]
        self.q_dev = [d[:q_el].view(run.Q[0].shape) for d in self.dev]
        self.kv_dev = [d[q_el:] for d in self.dev]
        self.out = [run.out, torch.empty_like(run.out)]
        self.copy_stream = torch.cuda.Stream(device=run.device)
        self.caches = torch.tensor([p for l in range(nL) for p in (run.K[l].data_ptr(), run.V[l].data_ptr())],
                                   dtype=torch.int64, device=run.device)
        self.ws = L.workspace(256, run.device)
        self.h_host = run.h.cpu().pin_memory() if run.h is not None else None
        self.h_dev = torch.empty_like(run.h[0]) if run.h is not None else None
        self.out_host = torch.empty(run.steps, *run.out.shape, dtype=torch.float32).pin_memory()
        self.h2d = (q_el + kv_el) * 2
        self.h2d_pred = self.h_host[0].numel() * 2 if self.h_host is not None else 0
        self.d2h = run.out.numel() * 4

    def bytes_per_run(self):
        r = self.run
        return self.h2d * r.steps + self.h2d_pred * r.n_pred, self.d2h * r.steps

    def body(self, stream):
        r, w = self.run, self.run.w
        cs = self.copy_stream
        n = r.steps
        in_ready = [torch.cuda.Event() for _ in range(n)]   # step i's inputs are on the device
        in_done = [torch.cuda.Event() for _ in range(n)]    # step i has read them (slot i % 2 free)
        out_ready = [torch.cuda.Event() for _ in range(n)]  # step i's outputs are written
        out_done = [torch.cuda.Event() for _ in range(n)]   # ... and copied to the host (slot i % 2 free)
        self._events = (in_ready, in_done, out_ready, out_done)

        def fetch(i):  # step i's inputs into slot i % 2, on the copy stream
            with torch.cuda.stream(cs):
                if i >= 2:
                    cs.wait_event(in_done[i - 2])
                self.dev[i % 2].copy_(self.host[i], non_blocking=True)
                in_ready[i].record(cs)

        cs.wait_stream(stream)
        fetch(0)
        for i in range(n):
            if i + 1 < n:
                fetch(i + 1)
            stream.wait_event(in_ready[i])
            if i >= 2:
                stream.wait_event(out_done[i - 2])
            L.kv_append(r.dec.dims, w.n_layers, self.kv_dev[i % 2], self.caches, r.dec.ctx[i], self.ws, stream)
            h = None
            if is_prediction_step(i, w.interval) and self.h_host is not None:
                self.h_dev.copy_(self.h_host[i // w.interval], non_blocking=True)
                h = self.h_dev
            qd = r.qp_direct[i // w.interval] if r.qp_direct is not None else None
            r.dec.step(i, self.q_dev[i % 2], self.out[i % 2], h=h, qp_direct=qd, stream=stream)
            in_done[i].record(stream)
            out_ready[i].record(stream)
            with torch.cuda.stream(cs):
                cs.wait_event(out_ready[i])
                self.out_host[i].copy_(self.out[i % 2], non_blocking=True)
                out_done[i].record(cs)
        stream.wait_stream(cs)


def replica(base: tb_inputs.Workload, rank: int) -> tb_inputs.Workload:
    """Rank `rank`'s independent replica: same shapes, its own seeded data."""
    return base.scaled(seed=base.seed + rank)


def max_over_ranks(value: float, device) -> float:
    """The largest `value` over all ranks (the job is as slow as its slowest
    rank); identity outside torch.distributed."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return value
    t = torch.tensor([value], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.item()


def aggregate_rate(world: int, units_per_rank_step: float, ms_per_step: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return world * units_per_rank_step / (ms_per_step / 1000.0)


def time_graph(g, warmup, steps, dist_on, device):
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        g.replay()
    t1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), device)
    if dist_on:
        torch.distributed.barrier()
    return ms


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.proc = subprocess.Popen(["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def profiled_traffic(kernel: str, workload: str, root: str = ROOT):
    """DRAM bytes per launch from the committed ncu capture of `kernel` on
    `workload`, or None when the record was taken on another workload, when any
    of that kernel's source files has changed since the capture, or when the
    record is missing."""
    import hashlib
    try:
        with open(os.path.join(root, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel]
        if rec.get("workload_name") != workload or not rec["sources"]:
            return None
        for path, sha in rec["sources"].items():
            with open(os.path.join(root, path), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != sha:
                    return None
        return rec["dram_read_bytes"] + rec["dram_write_bytes"]
    except (OSError, KeyError, TypeError, ValueError):
        return None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------------------
# CPU oracle on a bounded sample
# ----------------------------------------------------------------------------

def host_info() -> dict:
    """The host's logical core count and CPU model (for the CPU baseline)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu_model": model}


class OracleSample:
    """The oracle on one layer of the workload: the key projection of the
    prefilled context (setup, timed), then decode steps of that layer in
    schedule order.  A prediction step scores and selects for every query head
    from the layer's slot of its producer's predicted queries (the predictor
    MLP itself is timed apart, once per producer call); every step runs
    attention for every query head."""

    def __init__(self, w: tb_inputs.Workload, layer: int = 0):
        import numpy as np

        import oracle
        self.np, self.o = np, oracle
        self.w = w
        self.layer = layer
        K, V = tb_inputs.kv_layer(w, layer, "cpu")
        self.K = K.view(torch.int16).numpy().view(np.uint16)
        self.V = V.view(torch.int16).numpy().view(np.uint16)
        self.Wk = tb_inputs.wk_layer(w, layer, "cpu").view(torch.int16).numpy().view(np.uint16)
        self.ctx0 = w.ctx0_per_seq()
        self.scale = 1.0 / math.sqrt(w.head_dim)
        self.Kp = {}
        t0 = time.perf_counter()
        for b in range(w.batch):
            for g in range(w.n_kv_heads):
                n = (self.ctx0[b] // w.window) * w.window
                self.Kp[(b, g)] = self.o.project_keys(self.K[b, g, :n + w.window], self.Wk[g])
        self.proj_s = time.perf_counter() - t0
        self.rows_projected = sum((t // w.window) * w.window + w.window for t in self.ctx0) * w.n_kv_heads
        self.stride = w.producer_stride if w.hidden > 0 else 1
        self.producer = layer - layer % self.stride
        if w.hidden > 0:
            W1, W2 = tb_inputs.mlp_weights(w, self.producer, "cpu")
            self.W1 = W1.view(torch.int16).numpy().view(np.uint16)
            self.W2 = W2.view(torch.int16).numpy().view(np.uint16)
        self.I = None
        self.mlp_s = []

    def step(self, i):
        np, o, w = self.np, self.o, self.w
        ctx = [t + i + 1 for t in self.ctx0]
        if is_prediction_step(i, w.interval):
            if w.hidden > 0:
                h = tb_inputs.hidden_state(w, i // w.interval, self.producer, "cpu").view(torch.int16).numpy().view(
                    np.uint16)
                t0 = time.perf_counter()
                qp = o.predict_queries(h, self.W1, self.W2).reshape(w.batch, w.slots, w.n_q_heads, w.d_proj)
                self.mlp_s.append(time.perf_counter() - t0)
                qp = qp[:, self.layer % self.stride]
            else:
                qp = tb_inputs.direct_qp(w, i // w.interval, self.layer, "cpu").numpy()
            self.I = []
            for b in range(w.batch):
                T = ctx[b]
                hi = max(w.sink, T - w.window)
                per = []
                for h_ in range(w.n_q_heads):
                    s = o.scores(qp[b, h_], self.Kp[(b, h_ // w.group)], w.sink, hi)
                    per.append(o.select(s, T, w.sink, w.window, w.budget, w.nbr))
                self.I.append(per)
        Q = tb_inputs.query(w, i, self.layer, "cpu").view(torch.int16).numpy().view(np.uint16)
        for b in range(w.batch):
            for h_ in range(w.n_q_heads):
                A = o.attention_set(ctx[b], w.sink, w.window, self.I[b][h_])
                o.attention(Q[b, h_], self.K[b, h_ // w.group], self.V[b, h_ // w.group], A, self.scale)


def per_decode_step_s(w, layers: list[dict]) -> float:
    """Whole-model oracle seconds per decode step from per-layer samples.  Each
    sample holds the layer's mean prediction-step time (without the predictor
    MLP), mean reuse-step time, predictor MLP time (producer layers; None
    otherwise) and projection seconds per projected row.  Every layer pays
    attention at every step and scoring + selection once per interval; the
    predictor is paid once per producer layer per interval; key projection
    once per new token."""
    per_layer = statistics.mean((x["t_pred"] + (w.interval - 1) * x["t_reuse"]) / w.interval for x in layers)
    mlps = [x["t_mlp"] for x in layers if x["t_mlp"] is not None]
    n_prod = len(range(0, w.n_layers, w.producer_stride)) if w.hidden > 0 else 0
    mlp = (statistics.mean(mlps) * n_prod / w.interval) if mlps else 0.0
    proj_row = statistics.mean(x["proj_s_per_row"] for x in layers)
    rows_per_step = w.batch * w.n_kv_heads                     # one new row per (sequence, KV head)
    return w.n_layers * (per_layer + proj_row * rows_per_step) + mlp


def sample_layers(w) -> list[int]:
    return sorted({0, min(1, w.n_layers - 1), w.n_layers - 1})


def oracle_layer_sample(w, layer: int, budget_s: float) -> dict:
    """Time one layer: its projection setup, its first (prediction) step and
    reuse steps until `budget_s` seconds of steps have passed."""
    smp = OracleSample(w, layer)
    t_pred, t_reuse = [], []
    t_start = time.perf_counter()
    i = 0
    while i < w.steps:
        t0 = time.perf_counter()
        smp.step(i)
        dt = time.perf_counter() - t0
        if is_prediction_step(i, w.interval):
            t_pred.append(dt - (smp.mlp_s[-1] if smp.mlp_s else 0.0))
        else:
            t_reuse.append(dt)
        i += 1
        if t_reuse and time.perf_counter() - t_start > budget_s:
            break
    return {"layer": layer, "t_pred": statistics.mean(t_pred), "t_reuse": statistics.mean(t_reuse or t_pred),
            "t_mlp": statistics.mean(smp.mlp_s) if (smp.mlp_s and layer % smp.stride == 0) else None,
            "proj_s_per_row": smp.proj_s / smp.rows_projected, "setup_s": smp.proj_s,
            "n_pred": len(t_pred), "n_reuse": len(t_reuse)}


def cpu_baseline(w, budget_s=6.0):
    t0 = time.perf_counter()
    layers = [oracle_layer_sample(w, l, budget_s) for l in sample_layers(w)]
    s_per_step = per_decode_step_s(w, layers)
    desc = "; ".join(f"layer {x['layer']}: setup {x['setup_s']:.1f} s, {x['n_pred']} prediction + {x['n_reuse']} "
                     f"reuse steps" for x in layers)
    return dict({"value": w.batch / s_per_step, "unit": "decode steps/s", "cores": 1, "kind": "oracle",
                 "sample": (f"{w.name}, layers {[x['layer'] for x in layers]} of {w.n_layers}, every query head, "
                            f"one thread ({desc}); key projection of the prefilled context timed as setup and "
                            f"charged per new token; per-layer step times averaged over the sampled layers and "
                            f"scaled to all layers, selection amortised over the {w.interval}-step interval, the "
                            f"predictor MLP once per producer layer per interval"),
                 "sample_seconds": round(time.perf_counter() - t0, 1)}, **host_info())


def config_of(w: tb_inputs.Workload, decode_steps: int, world: int, selection: str = "head",
              sharded: bool = False) -> dict:
    """The workload description both arms print."""
    return {"workload": w.name, "batch": w.batch, "ctx": w.ctx0 if not w.ragged else [w.ctx0_lo, w.ctx0_hi],
            "layers": w.n_layers, "decode_steps_per_bench_step": decode_steps, "budget": w.budget,
            "interval": w.interval, "sink": w.sink, "window": w.window, "d_proj": w.d_proj,
            "selection": {"head": "per query head", "inclusive": "per query head, budget includes neighbours"}.get(
                selection, f"per KV head ({selection})"),
            "parallelism": (f"kv-head shards x{world}" if sharded else f"replicas x{world}") if world > 1
            else "single GPU"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = tb_inputs.WORKLOADS[args.workload]
    layers = sample_layers(w)
    samples = {l: OracleSample(w, l) for l in layers}
    for smp in samples.values():
        for i in range(min(args.warmup, w.steps)):     # step 0 predicts, so reuse steps have a selection
            smp.step(i)
    t_all0 = time.perf_counter()
    per = {l: {"pred": [], "reuse": []} for l in layers}
    for k in range(args.steps):
        # each bench step: one decode step of every sampled layer, cycling
        # through the schedule so prediction steps come in their proportion
        i = k % w.steps
        for l, smp in samples.items():
            t0 = time.perf_counter()
            smp.step(i)
            dt = time.perf_counter() - t0
            if is_prediction_step(i, w.interval):
                per[l]["pred"].append(dt - (smp.mlp_s[-1] if smp.mlp_s else 0.0))
            else:
                per[l]["reuse"].append(dt)
    wall = time.perf_counter() - t_all0
    stats = []
    for l, smp in samples.items():
        pr, ru = per[l]["pred"], per[l]["reuse"]
        if not pr:                                       # no prediction step timed: the warm-up one
            smp_w = OracleSample(w, l)
            t0 = time.perf_counter()
            smp_w.step(0)
            pr = [time.perf_counter() - t0 - (smp_w.mlp_s[-1] if smp_w.mlp_s else 0.0)]
            smp = smp_w
        stats.append({"layer": l, "t_pred": statistics.mean(pr), "t_reuse": statistics.mean(ru or pr),
                      "t_mlp": statistics.mean(smp.mlp_s) if (smp.mlp_s and l % smp.stride == 0) else None,
                      "proj_s_per_row": smp.proj_s / smp.rows_projected})
    value = w.batch / per_decode_step_s(w, stats)
    sample = (f"each bench step: one decode step of layers {layers} of {w.name} (all {w.n_q_heads} query heads, one "
              f"thread), in schedule order; per-layer times scaled to {w.n_layers} layers with selection amortised "
              f"over the {w.interval}-step interval, the predictor once per producer layer")
    cb = dict({"value": round(value, 4), "unit": "decode steps/s", "cores": 1, "kind": "oracle", "sample": sample},
              **host_info())
    line = {"impl": "reference", "metric": "sparse decode steps/s", "value": round(value, 4),
            "unit": "decode steps/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1000 * wall / max(1, args.steps), 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, args.decode_steps or w.steps, args.gpus),
            "cpu_baseline": cb,
            "e2e": {"value": round(value, 4), "unit": "decode steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------------------
# main
# ----------------------------------------------------------------------------

def measure(w, args, device, dist_on, world, with_e2e: bool, steps: int, warmup: int, selection: str,
            shard=None):
    """Time one workload's sparse run, dense run and (optionally) the e2e run,
    each replayed as one CUDA graph; returns the figures the JSON line needs.
    With shard=(rank, world) this rank runs only its KV heads of the one
    workload (strong scaling: the job's tokens are the workload's tokens)."""
    run = Run(w, device, steps=args.decode_steps, selection=selection, shard=shard, balance=not args.no_balance,
              overlap_select=not args.no_overlap, select_streams=args.select_streams)
    copies = 1 if shard else world          # independent replicas count every rank's tokens
    run.dec.prefill()
    torch.cuda.synchronize()

    acct = run.bytes_model()       # eager pass: warms every kernel and counts the kept rows
    stream = torch.cuda.Stream(device=device)
    marks_s = Marks(run.steps)
    marks_s.stream = stream
    g_sparse = capture(lambda st: run.run_sparse(st, marks_s), stream, count_kernels=True)
    marks_d = Marks(run.steps)
    marks_d.stream = stream
    g_dense = capture(lambda st: run.run_dense(st, marks_d), stream)
    e2e = g_e2e = None
    if with_e2e:
        e2e = E2E(run)
        g_e2e = capture(e2e.body, stream)
    torch.cuda.synchronize()

    clocks = ClockSampler(torch.cuda.current_device())
    ms_sparse = time_graph(g_sparse, warmup, steps, dist_on, device)
    attn_ms = marks_s.attn_ms(run.steps)
    ms_dense = time_graph(g_dense, warmup, steps, dist_on, device)
    dense_attn_ms = marks_d.attn_ms(run.steps)
    clk = clocks.stop()
    ms_e2e = clk_e2e = None
    if e2e is not None:
        clocks = ClockSampler(torch.cuda.current_device())
        ms_e2e = time_graph(g_e2e, warmup, steps, dist_on, device)
        clk_e2e = clocks.stop()

    flags = 0
    for ws in run.dec.workspaces():
        flags |= L.workspace_check(ws)

    tokens_per_run = run.steps * w.batch
    per_step_sparse = ms_sparse / steps
    per_step_dense = ms_dense / steps
    n_attn = run.steps * w.n_layers
    attn_launch_ms = sum(attn_ms) / n_attn
    dense_launch_ms = sum(dense_attn_ms) / n_attn
    res = dict(
        run_steps=run.steps, tokens_per_run=tokens_per_run, acct=acct,
        value=aggregate_rate(copies, tokens_per_run, per_step_sparse),
        dense_value=aggregate_rate(copies, tokens_per_run, per_step_dense),
        per_step_sparse=per_step_sparse, per_step_dense=per_step_dense,
        attn_launch_ms=attn_launch_ms, attn_bytes_per_launch=acct["attn_bytes"] / n_attn,
        dense_launch_ms=dense_launch_ms, dense_bytes_per_launch=(acct["dense_total"] / n_attn),
        path_gbs=acct["sparse_total"] / (per_step_sparse / 1000.0) / 1e9,
        dense_path_gbs=acct["dense_total"] / (per_step_dense / 1000.0) / 1e9,
        launches=g_sparse.libtb_kernels, clocks=clk, flags=flags,
        kv_gb=2 * sum(k.numel() for k in run.K) * 2 / 1e9)
    if e2e is not None:
        h2d, d2h = e2e.bytes_per_run()
        res["e2e"] = {"value": round(aggregate_rate(copies, tokens_per_run, ms_e2e / steps), 3),
                      "unit": "decode steps/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                      "ms_per_step": round(ms_e2e / steps, 4), "clocks": clk_e2e}
    del g_sparse, g_dense, g_e2e, e2e, run
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def measure_offload(w, args, device, selection: str):
    """Per-token decode latency with the KV cache in pinned host memory (the
    CPU-offloading workload): the sparse path against dense attention over the
    same host cache.  The prediction step, a reuse step, a projection step and
    a dense step are each captured as a graph and timed apart; the sparse
    per-token latency amortises prediction over the interval and projection
    over its N-token batch."""
    N, P = w.window, w.interval
    steps = max(P, N)                                       # the first projection batch falls at step < N
    run = Run(w, device, steps=steps, selection=selection, offload=True)
    run.dec.prefill()
    torch.cuda.synchronize()
    t_off = time.perf_counter()
    run.dec.offload()
    run.K = run.V = None
    torch.cuda.empty_cache()
    t_off = time.perf_counter() - t_off
    proj_step = run.dec.proj_steps[0] if run.dec.proj_steps else None
    stream = torch.cuda.Stream(device=device)

    def one(i, dense=False):
        Q, h, qd = run.step_inputs(i)
        if dense:
            return capture(lambda st: run.dec.dense_step(i, Q, run.out, stream=st), stream)
        return capture(lambda st: run.dec.step(i, Q, run.out, h=h, qp_direct=qd, stream=st), stream)

    for i in (0, 1):                                        # eager: every kernel warmed, the sets in place
        Q, h, qd = run.step_inputs(i)
        run.dec.step(i, Q, run.out, h=h, qp_direct=qd)
    torch.cuda.synchronize()
    graphs = {"pred": one(0), "reuse": one(1), "dense": one(1, dense=True)}
    if proj_step is not None and not is_prediction_step(proj_step, P):
        graphs["proj"] = one(proj_step)
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device())
    ms = {k: time_graph(g, max(3, args.warmup), args.extra_steps, False, device) / args.extra_steps
          for k, g in graphs.items()}
    clk = clocks.stop()
    flags = 0
    for ws in run.dec.workspaces():
        flags |= L.workspace_check(ws)
    sparse_ms = (ms["pred"] + (P - 1) * ms["reuse"]) / P + ((ms["proj"] - ms["reuse"]) / N if "proj" in ms else 0.0)
    host_gb = sum(hb.nbytes for hb in run.dec.K_host + run.dec.V_host) / 1e9
    res = {"workload": w.name, "per_token_ms": round(sparse_ms, 3), "dense_per_token_ms": round(ms["dense"], 3),
           "speedup_vs_dense": round(ms["dense"] / sparse_ms, 3),
           "step_ms": {k: round(v, 3) for k, v in ms.items()},
           "host_kv_gb": round(host_gb, 2), "offload_s": round(t_off, 1), "clocks": clk, "device_flags": flags,
           "note": ("K and V in pinned host memory read by the attention kernels across the host link; K', "
                    "the predictor, scoring and selection on the device; per-token = (prediction step + "
                    f"{P - 1} reuse steps)/{P} + (projection step - reuse step)/{N}")}
    for hb in run.dec.K_host + run.dec.V_host:
        hb.free()
    del graphs, run
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def summary(w, r, peak):
    """The compact per-workload figures of the extra workloads."""
    achieved = r["attn_bytes_per_launch"] / (r["attn_launch_ms"] / 1000.0) / 1e9
    return {"value": round(r["value"], 3), "unit": "decode steps/s", "ms_per_step": round(r["per_step_sparse"], 4),
            "dense_value": round(r["dense_value"], 3), "speedup_vs_dense": round(r["value"] / r["dense_value"], 4),
            "path_gbs": round(r["path_gbs"], 1), "path_frac_of_8tbs": round(r["path_gbs"] / HBM_NOMINAL_GBS, 4),
            "attn_achieved_gbs": round(achieved, 1), "attn_frac": round(achieved / peak, 4),
            "attn_launch_us": round(1000 * r["attn_launch_ms"], 3),
            "dense_attn_frac": round(r["dense_bytes_per_launch"] / (r["dense_launch_ms"] / 1000.0) / 1e9 / peak, 4),
            "decode_steps_per_bench_step": r["run_steps"], "clocks": r["clocks"], "device_flags": r["flags"],
            "config": {"batch": w.batch, "ctx": w.ctx0 if not w.ragged else [w.ctx0_lo, w.ctx0_hi],
                       "layers": w.n_layers, "budget": w.budget, "interval": w.interval,
                       "kv_gb": round(r["kv_gb"], 1)}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=6)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama64k", choices=sorted(tb_inputs.WORKLOADS))
    ap.add_argument("--impl", default="tb", choices=["tb", "reference"])
    ap.add_argument("--decode-steps", type=int, default=None, help="decode steps per run (default: workload's)")
    ap.add_argument("--layers", type=int, default=None, help="override the layer count (profiling runs)")
    ap.add_argument("--interval", type=int, default=None,
                    help="override the prediction interval P (1: predict and select at every step)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the extra workloads (batch16, long256k, llama64k at interval 1) timed after the "
                         "headline one")
    ap.add_argument("--extra-steps", type=int, default=3, help="timed bench steps of each extra workload")
    ap.add_argument("--no-offload", action="store_true",
                    help="skip the CPU-offloaded KV cache on long256k (per-token latency against dense), which the "
                         "default single-GPU run times after the headline workload")
    ap.add_argument("--offload-only", action="store_true", help="time only the CPU-offloaded workload")
    ap.add_argument("--no-overlap", action="store_true",
                    help="all of a prediction step's selections on one stream (no extra selection streams)")
    ap.add_argument("--select-streams", type=int, default=4,
                    help="streams a prediction step's selections go round-robin over (with the overlap on)")
    ap.add_argument("--no-balance", action="store_true",
                    help="attention slices at equal shares of the length instead of the kept rows (no tb_attn_plan)")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "kv_heads"],
                    help="with N > 1 ranks: replicas (each rank decodes its own seeded replica; weak scaling) or "
                         "kv_heads (the ranks split one workload's KV heads; strong scaling)")
    ap.add_argument("--selection", default="head", choices=list(SparseDecoder.SELECTIONS),
                    help="head: one importance set per query head (the default, the pages' reading); "
                         "group_max / group_sum: one set per KV head (the group-shared variant); "
                         "inclusive: at most B positions per head after neighbour fetch")
    args = ap.parse_args()

    if args.impl == "reference":
        return run_reference(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = f"cuda:{local}"
    dist_on = world > 1
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device(device))
    L.load()

    sharded = args.shard == "kv_heads"
    shard = (rank, world) if sharded else None

    def prepare(name):
        # an independent replica per rank, or one workload split by KV heads
        w = tb_inputs.WORKLOADS[name] if sharded else replica(tb_inputs.WORKLOADS[name], rank)
        if args.layers:
            w = w.scaled(n_layers=args.layers)
        if args.interval:
            w = w.scaled(interval=args.interval)
        return w

    if args.offload_only:
        print(json.dumps({"offload": measure_offload(prepare("long256k"), args, device, args.selection)}))
        return 0
    w = prepare(args.workload)
    r = measure(w, args, device, dist_on, world, not args.no_e2e, args.steps, args.warmup, args.selection, shard)
    extras = {}
    if not args.no_extra and args.workload == "llama64k" and not args.layers and not args.decode_steps:
        # the other two large workloads, each against the dense kernel on its own cache
        for name in ("long256k", "batch16"):
            wx = prepare(name)
            extras[name] = summary(wx, measure(wx, args, device, dist_on, world, False, args.extra_steps,
                                               max(3, args.warmup), args.selection, shard), measured_peaks()[0])
        # the headline workload with a prediction (and selection) at every
        # decode step: what the interval amortises
        wx = prepare("llama64k").scaled(interval=1)
        extras["llama64k_interval1"] = summary(wx, measure(wx, args, device, dist_on, world, False, args.extra_steps,
                                                           max(3, args.warmup), args.selection, shard),
                                               measured_peaks()[0])

    offload = None
    # (a per-token latency on one GPU: not run under torchrun, where every
    # rank would pin its own 34 GB copy of the cache in host memory)
    if not args.no_offload and args.workload == "llama64k" and not args.layers and not args.decode_steps and \
            world == 1:
        try:
            offload = measure_offload(prepare("long256k"), args, device, args.selection)
        except (RuntimeError, MemoryError) as e:   # e.g. the host cannot pin 34 GB
            offload = {"workload": "long256k", "unavailable": str(e).splitlines()[0][:200]}
    peak, peak_kind = measured_peaks()
    acct = r["acct"]
    achieved = r["attn_bytes_per_launch"] / (r["attn_launch_ms"] / 1000.0) / 1e9
    dense_achieved = r["dense_bytes_per_launch"] / (r["dense_launch_ms"] / 1000.0) / 1e9

    if rank != 0:
        if dist_on:
            torch.distributed.destroy_process_group()
        return 0
    line = {
        "metric": "sparse decode steps/s", "value": round(r["value"], 3), "unit": "decode steps/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(r["per_step_sparse"], 4),
        "higher_is_better": True, "scaling": "strong" if sharded else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; Llama-3.1-8B attention shapes, random weights)",
        "config": dict(config_of(w, r["run_steps"], world, args.selection, sharded),
                       l2="inputs larger than L2 (KV %.1f GB)" % r["kv_gb"],
                       graph="one CUDA graph per bench step"),
        "speedup_vs_dense": round(r["value"] / r["dense_value"], 4),
        "dense": {"value": round(r["dense_value"], 3), "unit": "decode steps/s",
                  "ms_per_step": round(r["per_step_dense"], 4), "path_gbs": round(r["dense_path_gbs"], 1),
                  "attn_launch_us": round(1000 * r["dense_launch_ms"], 3),
                  "attn_achieved_gbs": round(dense_achieved, 1)},
        "hbm": {"path_gbs": round(r["path_gbs"], 1), "path_frac_of_8tbs": round(r["path_gbs"] / HBM_NOMINAL_GBS, 4),
                "path_frac_of_measured": round(r["path_gbs"] / peak, 4), "bytes_per_bench_step": acct["sparse_total"],
                "attn_rows_union": acct["attn_rows"], "attn_rows_per_head_sum": acct["sum_head_rows"],
                "dense_bytes_per_bench_step": acct["dense_total"]},
        "roofline": {"kernel": "attn_kernel<128,true> (sparse GQA decode attention)", "bound": "hbm",
                     "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": (profiled_traffic("attn_kernel<128,true>", w.name)
                                 if args.selection == "head" and not args.layers and not args.interval else None),
                     "bytes_per_launch": round(r["attn_bytes_per_launch"]),
                     "launch_us": round(1000 * r["attn_launch_ms"], 3)},
        "gpu_launches": r["launches"] * args.steps,
        "clocks": r["clocks"],
        "device_flags": r["flags"],
    }
    if "e2e" in r:
        line["e2e"] = r["e2e"]
    if extras:
        line["workloads"] = extras
    if offload:
        line["offload"] = offload
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line))
    if dist_on:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
