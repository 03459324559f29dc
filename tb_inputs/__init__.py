"""Seeded synthetic inputs for the TokenButler decode path.

This module is shared by the CUDA path (tests, benchmark) and by the oracle
side of the tests.  It only draws random numbers and lays them out; it holds
none of the method's arithmetic (no projection, scoring, selection or
attention).

Workloads (sizes follow the Llama-3.1-8B attention shape the TokenButler
summaries evaluate on: 32 query heads, 8 KV heads, head_dim 128, hidden 4096):

  tiny300     1 sequence, 1 layer, 8/2 heads, d=64, context 300, d'=16,
              S=4, N=16, B=32, one decode step, integer values in [-4, 4]
  llama8k     1 layer, context 8192, MLP 4096->1024->32x32, B=1024,
              interval 16 over 64 steps
  llama64k    32 layers, context 65536, producer every 4 layers, B=8192,
              interval 16 over 256 steps, 1% planted heavy-hitter keys (x4)
  batch16     32 layers, 16 sequences with contexts uniform in [16384, 32768],
              B=2048, interval 8 over 128 steps
  long256k    32 layers, context 262144, B=8192, interval 16 over 64 steps,
              planted heavy hitters

Value recipe: K, V, Q, h ~ N(0, 1); W1, W2, W_k ~ N(0, 0.02) (all stored
bf16); the tiny case draws every input, including q', as integers uniform on
[-4, 4].  Every tensor has its own generator seeded from (workload seed,
tensor name, indices), so any layer can be regenerated alone.
"""
from __future__ import annotations

import dataclasses
import hashlib
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    d_proj: int
    hidden: int            # 0: q' is drawn directly, no predictor MLP
    inter: int
    producer_stride: int   # producer layers are l % stride == 0; slots G = stride
    ctx0: int              # prefilled tokens (fixed contexts)
    ctx0_lo: int           # ragged contexts: uniform in [ctx0_lo, ctx0_hi]
    ctx0_hi: int
    sink: int
    window: int
    budget: int
    nbr: int
    interval: int
    steps: int
    integer_valued: bool = False
    heavy_frac: float = 0.0
    heavy_scale: float = 4.0
    w_std: float = 0.02
    seed: int = 0

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def slots(self) -> int:
        """G: query slots emitted per producer call (one per served layer)."""
        return self.producer_stride

    @property
    def n_out(self) -> int:
        return self.slots * self.n_q_heads * self.d_proj

    @property
    def ragged(self) -> bool:
        return self.ctx0_hi > self.ctx0_lo

    def ctx0_per_seq(self) -> list[int]:
        if not self.ragged:
            return [self.ctx0] * self.batch
        g = torch.Generator().manual_seed(_seed(self, "ctx0"))
        v = torch.randint(self.ctx0_lo, self.ctx0_hi + 1, (self.batch,), generator=g)
        return [int(x) for x in v]

    @property
    def ctx_cap(self) -> int:
        """Row capacity per (sequence, KV head): longest prefill + decode steps,
        rounded up to a multiple of 128."""
        t = max(self.ctx0_per_seq()) + self.steps
        return (t + 127) // 128 * 128

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny300": Workload("tiny300", batch=1, n_layers=1, n_q_heads=8, n_kv_heads=2,
                        head_dim=64, d_proj=16, hidden=0, inter=0, producer_stride=1,
                        ctx0=299, ctx0_lo=299, ctx0_hi=299, sink=4, window=16,
                        budget=32, nbr=1, interval=1, steps=1, integer_valued=True),
    "llama8k": Workload("llama8k", batch=1, n_layers=1, n_q_heads=32, n_kv_heads=8,
                        head_dim=128, d_proj=32, hidden=4096, inter=1024, producer_stride=1,
                        ctx0=8192, ctx0_lo=8192, ctx0_hi=8192, sink=16, window=64,
                        budget=1024, nbr=1, interval=16, steps=64),
    "llama64k": Workload("llama64k", batch=1, n_layers=32, n_q_heads=32, n_kv_heads=8,
                         head_dim=128, d_proj=32, hidden=4096, inter=1024, producer_stride=4,
                         ctx0=65536, ctx0_lo=65536, ctx0_hi=65536, sink=16, window=64,
                         budget=8192, nbr=1, interval=16, steps=256, heavy_frac=0.01),
    "batch16": Workload("batch16", batch=16, n_layers=32, n_q_heads=32, n_kv_heads=8,
                        head_dim=128, d_proj=32, hidden=4096, inter=1024, producer_stride=4,
                        ctx0=0, ctx0_lo=16384, ctx0_hi=32768, sink=16, window=64,
                        budget=2048, nbr=1, interval=8, steps=128),
    "long256k": Workload("long256k", batch=1, n_layers=32, n_q_heads=32, n_kv_heads=8,
                         head_dim=128, d_proj=32, hidden=4096, inter=1024, producer_stride=4,
                         ctx0=262144, ctx0_lo=262144, ctx0_hi=262144, sink=16, window=64,
                         budget=8192, nbr=1, interval=16, steps=64, heavy_frac=0.01),
}


def _seed(w: Workload, *keys) -> int:
    h = hashlib.sha256(repr((w.name, w.seed) + tuple(keys)).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(w: Workload, device, *keys) -> torch.Generator:
    return torch.Generator(device=device).manual_seed(_seed(w, *keys))


def _draw(w: Workload, shape, device, std: float, *keys) -> torch.Tensor:
    g = _gen(w, device, *keys)
    if w.integer_valued:
        x = torch.randint(-4, 5, shape, generator=g, device=device, dtype=torch.int32)
        return x.to(torch.bfloat16)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def kv_layer(w: Workload, layer: int, device="cpu") -> tuple[torch.Tensor, torch.Tensor]:
    """K, V of one layer, [batch][Hkv][ctx_cap][d] bf16.  Rows past a sequence's
    final length (prefill + steps) are zero.  Rows at decode positions hold the
    tokens the decode loop appends, drawn in advance."""
    shape = (w.batch, w.n_kv_heads, w.ctx_cap, w.head_dim)
    K = _draw(w, shape, device, 1.0, "K", layer)
    V = _draw(w, shape, device, 1.0, "V", layer)
    if w.heavy_frac > 0:
        n_heavy = max(1, int(round(w.heavy_frac * w.ctx_cap)))
        for b in range(w.batch):
            for g in range(w.n_kv_heads):
                gen = _gen(w, "cpu", "heavy", layer, b, g)
                pos = torch.randperm(w.ctx_cap, generator=gen)[:n_heavy].to(device)
                K[b, g, pos, :] = K[b, g, pos, :] * w.heavy_scale
    ends = [t + w.steps for t in w.ctx0_per_seq()]
    for b, e in enumerate(ends):
        if e < w.ctx_cap:
            K[b, :, e:, :] = 0
            V[b, :, e:, :] = 0
    return K, V


def wk_layer(w: Workload, layer: int, device="cpu") -> torch.Tensor:
    """W_k of one layer, [Hkv][d'][d] bf16 (output-major)."""
    return _draw(w, (w.n_kv_heads, w.d_proj, w.head_dim), device, w.w_std, "Wk", layer)


def mlp_weights(w: Workload, producer: int, device="cpu") -> tuple[torch.Tensor, torch.Tensor]:
    """W1 [inter][hidden], W2 [G*Hq*d'][inter] (bf16) of one producer layer."""
    W1 = _draw(w, (w.inter, w.hidden), device, w.w_std, "W1", producer)
    W2 = _draw(w, (w.n_out, w.inter), device, w.w_std, "W2", producer)
    return W1, W2


def hidden_state(w: Workload, pred_step: int, producer: int, device="cpu") -> torch.Tensor:
    """Producer-layer hidden state at a prediction step, [batch][hidden] bf16."""
    return _draw(w, (w.batch, w.hidden), device, 1.0, "h", pred_step, producer)


def direct_qp(w: Workload, pred_step: int, layer: int, device="cpu") -> torch.Tensor:
    """q' drawn directly (workloads without a predictor), [batch][Hq][d'] fp32."""
    return _draw(w, (w.batch, w.n_q_heads, w.d_proj), device, 1.0, "qp", pred_step,
                 layer).to(torch.float32)


def query(w: Workload, step: int, layer: int, device="cpu") -> torch.Tensor:
    """Decode query of one step and layer, [batch][Hq][d] bf16."""
    return _draw(w, (w.batch, w.n_q_heads, w.head_dim), device, 1.0, "Q", step, layer)


def selection_sets(w: Workload, T: list[int], density: float, device="cpu", key=0):
    """Random importance sets for attention-only tests: for each (sequence,
    query head) a sorted set of candidate positions [S, T-N) of the given
    density.  Returned as a list (per sequence) of lists (per head) of int32
    tensors on the CPU."""
    out = []
    for b in range(w.batch):
        lo, hi = w.sink, T[b] - w.window
        heads = []
        for h in range(w.n_q_heads):
            if hi <= lo:
                heads.append(torch.zeros(0, dtype=torch.int32))
                continue
            g = _gen(w, "cpu", "sets", key, b, h)
            m = torch.rand(hi - lo, generator=g) < density
            heads.append((torch.nonzero(m).flatten() + lo).to(torch.int32))
        out.append(heads)
    return out
