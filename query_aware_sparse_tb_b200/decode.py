"""Decode-loop driver for the TokenButler path on device-resident buffers.

The schedule (TokenButler technical summary, gist.science):
  * "Core architecture": queries are predicted at producer layers placed at a
    fixed depth stride and consumed by the following layers; each producer
    call emits G slot-specific queries per head (here G = stride and slot j
    serves layer p + j).
  * "Optimisations: batching": keys are projected in batches of N tokens, not
    at every step (N = the local window, so every candidate [S, T-N) always
    has a projected key).
  * "Optimisations: prediction interval and neighbour fetch": the predictor,
    and with it scoring and selection, runs once every P steps; the selection
    is reused unchanged in between, while sink and window follow the current
    length.

Every step of the path runs in libtb's CUDA kernels; this module only decides
which entry point runs when, on which buffers, and can record a whole run into
one CUDA graph.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass

import torch

from . import _lib as L


def main_stream_last_selected(n_layers: int, n_streams: int) -> int:
    """The last layer whose selection the caller's stream issues when a
    prediction step's selections go round-robin over n_streams streams (layer
    l on stream l mod n_streams, the caller's stream first)."""
    return (n_layers - 1) // n_streams * n_streams


def is_prediction_step(step: int, interval: int) -> bool:
    return step % interval == 0


def producer_layer(layer: int, stride: int) -> int:
    return layer - layer % stride


def query_slot(layer: int, stride: int) -> int:
    return layer % stride


def projection_schedule(ctx0: list[int], window: int, steps: int):
    """Prefill lengths and per-step projection batches.

    Returns (prefill, events) where prefill[b] = floor(ctx0[b]/N)*N rows are
    projected before decoding, and events maps a step index to a list of
    per-sequence batch starts (-1 = this sequence projects nothing at that
    step).  A sequence projects its next N rows at the first step whose length
    T = ctx0 + step + 1 is N past its projected prefix."""
    prefill = [(t // window) * window for t in ctx0]
    proj = list(prefill)
    events: dict[int, list[int]] = {}
    for i in range(steps):
        begins = [-1] * len(ctx0)
        for b, t0 in enumerate(ctx0):
            if t0 + i + 1 - proj[b] >= window:
                begins[b] = proj[b]
                proj[b] += window
        if any(x >= 0 for x in begins):
            events[i] = begins
    return prefill, events


# --------------------------------------------------------------- KV-head sharding
#
# Tensor-parallel placement of the path: rank r of `world` owns a contiguous
# block of KV heads and the query heads of their GQA groups, with those heads'
# K, V, K' and W_k, and the rows of the predictor's second matrix that emit
# their queries (the first matrix is replicated: every rank needs the whole
# activation).  Projection, prediction, scoring, selection and attention are
# independent per head, so a rank runs the unchanged entry points on its slice
# and nothing crosses ranks on the way; the heads' outputs meet again only in
# the model's output projection (a TP all-reduce outside this path), or in an
# all-gather when the full [batch][Hq][d] output is wanted on every rank.

def kv_head_shard(n_kv_heads: int, group: int, rank: int, world: int) -> tuple[range, range]:
    """(KV heads, query heads) owned by `rank` of `world`: contiguous blocks."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if n_kv_heads % world:
        raise ValueError(f"{n_kv_heads} KV heads do not split over {world} ranks")
    per = n_kv_heads // world
    g0 = rank * per
    return range(g0, g0 + per), range(g0 * group, (g0 + per) * group)


def shard_w2(W2, slots: int, n_q_heads: int, d_proj: int, heads: range):
    """Rows of the predictor's second matrix W2 [slots*Hq*d'][inter] that emit
    the queries of `heads`, for every slot, in the [slot][head][d'] order of a
    predictor whose output has len(heads) heads."""
    inter = W2.shape[-1]
    return W2.reshape(slots, n_q_heads, d_proj, inter)[:, heads.start:heads.stop].reshape(-1, inter).contiguous()


def gather_head_outputs(parts, heads_of_rank):
    """Reassemble [..][batch][Hq][d] from the ranks' [..][batch][Hq_local][d]
    outputs (parts[r] holds rank r's query heads heads_of_rank[r])."""
    import torch
    order = sorted(range(len(parts)), key=lambda r: heads_of_rank[r].start)
    return torch.cat([parts[r] for r in order], dim=-2)


# --------------------------------------------------------------- context sharding
#
# One sequence's context split over ranks by position (the scale-out for
# contexts past what one device should hold): rank r keeps the K, V and K'
# rows of block [begin_r, end_r).  Each rank selects its block's local top-B,
# the ranks exchange those candidates, every rank merges them into the global
# selection (the global top-B is contained in the union of the blocks' top-B),
# attends over its block's share of sink, window and selected rows, and the
# ranks' unnormalised softmax states are combined.  The result is the
# single-device result; tb.h (context-parallel selection and attention) has
# the contract of each call.

def context_blocks(ctx_cap: int, world: int, window: int) -> list[tuple[int, int]]:
    """[begin, end) of each rank's block: equal blocks of whole windows (so
    every block starts on a 32-position word and on a projection batch), the
    last rank keeping everything from its begin to ctx_cap (where decoding
    appends)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    unit = window * 32 // math.gcd(window, 32)
    per = max(unit, (ctx_cap // world) // unit * unit)
    bounds = []
    for r in range(world):
        b0 = min(r * per, ctx_cap)
        b1 = ctx_cap if r == world - 1 else min((r + 1) * per, ctx_cap)
        bounds.append((b0, b1))
    return bounds


def block_capacity(block: tuple[int, int], window: int) -> int:
    """Rows a rank's local caches hold: its block plus one window, the rows a
    local selection may count as its window and never reads."""
    return block[1] - block[0] + window


def local_selection_params(T: int, block: tuple[int, int], sink: int, window: int) -> tuple[int, int]:
    """(local T, local sink) for a selection over the block's part of the
    candidates C = [sink, T - window): with window unchanged, the local
    candidates [local sink, local T - window) are C ∩ block in local rows."""
    b0, b1 = block
    local_T = max(1, min(T, b1 + window) - b0)
    return local_T, max(0, sink - b0)


def local_rows(T: int, block: tuple[int, int]) -> int:
    """Rows of the block that exist at length T (at least 1 for the call)."""
    return max(1, min(T, block[1]) - block[0])


class ContextShard:
    """One rank's block of a context-sharded layer: its K, V (and K') rows,
    the selection and attention workspaces, and the three phases of a
    prediction step.  `exchange` between the phases is the caller's (an
    all-gather over the ranks; stacking the ranks' tensors on one device
    emulates it).  Per-head selection, queries given directly (q' of the
    block's sequences, [batch][Hq][d']).

      cand = shard.select_local(T, qp)              phase 1: local top-B
      part = shard.merge_and_attend(T, cands, Q)    phase 2: global set, partial attention
      combine_parts(parts, out)                     phase 3
    """

    def __init__(self, shape: "DecodeShape", block: tuple[int, int], K, V, Wk, device="cuda"):
        s = self.shape = shape
        self.block = block
        self.cap = block_capacity(block, s.window)
        assert K.shape[2] == self.cap and V.shape[2] == self.cap, "local caches hold block_capacity rows"
        self.K, self.V, self.Wk = K, V, Wk
        self.device = device
        B, Hq, Hkv = s.batch, s.n_q_heads, s.n_kv_heads
        self.dims = L.dims(B, Hq, Hkv, s.head_dim, s.d_proj, self.cap)
        self.gdims = L.dims(B, Hq, Hkv, s.head_dim, s.d_proj, s.ctx_cap)
        self.Kp = torch.zeros(B, Hkv, self.cap, s.d_proj, dtype=torch.bfloat16, device=device)
        self.ws_sel = L.workspace(L.score_select_workspace_bytes(self.dims), device)
        self.ws_attn = L.workspace(L.attn_workspace_bytes(self.dims), device)
        self.ws_small = L.workspace(256, device)
        self.local_idx = torch.zeros(B, Hq, min(s.budget, self.cap), dtype=torch.int32, device=device)
        self.local_cnt = torch.zeros(B, Hq, dtype=torch.int32, device=device)
        self.local_bits = torch.zeros(B, Hq, (self.cap + 31) // 32, dtype=torch.int32, device=device)
        self.cand = torch.zeros(B, Hq, s.budget, dtype=torch.int64, device=device)
        self.idx = torch.zeros(B, Hq, s.idx_cap, dtype=torch.int32, device=device)
        self.cnt = torch.zeros(B, Hq, dtype=torch.int32, device=device)
        self.bits = torch.zeros(B, Hq, (self.cap + 31) // 32, dtype=torch.int32, device=device)
        self.part = torch.zeros(B, Hq, s.head_dim + 2, dtype=torch.float32, device=device)
        self.scale = 1.0 / math.sqrt(s.head_dim)

    def project(self, rows: list[int], stream=None):
        """Project the first rows[b] local rows of every sequence."""
        zero = torch.zeros(self.shape.batch, dtype=torch.int32, device=self.device)
        cnt = torch.tensor(rows, dtype=torch.int32, device=self.device)
        L.project_keys(self.dims, self.K, self.Wk, self.Kp, zero, cnt, max(max(rows), 1), self.ws_small, stream)

    def select_local(self, T: list[int], qp, stream=None):
        """Phase 1: this block's top-B per head (nbr = 0) as exchangeable
        (score key, global position) candidates [batch][Hq][budget]."""
        s = self.shape
        params = [local_selection_params(t, self.block, s.sink, s.window) for t in T]
        sinks = {p[1] for p in params}
        assert len(sinks) == 1
        self.sel_ctx = torch.tensor([p[0] for p in params], dtype=torch.int32, device=self.device)
        L.score_select(self.dims, qp, s.n_q_heads * s.d_proj, self.Kp, self.sel_ctx, sinks.pop(), s.window,
                       s.budget, 0, self.local_idx, self.local_cnt, self.local_bits, self.ws_sel, stream)
        L.select_export_candidates(self.dims, self.ws_sel, self.local_idx, self.local_cnt, s.budget, self.block[0],
                                   self.cand, stream)
        return self.cand

    def merge_and_attend(self, T: list[int], cands, Q, stream=None):
        """Phase 2: the global selection from every rank's candidates
        ([world][batch][Hq][budget]) and this block's unnormalised attention
        state [batch][Hq][d+2]."""
        s = self.shape
        self.ctx_g = torch.tensor(T, dtype=torch.int32, device=self.device)
        self.rows = torch.tensor([local_rows(t, self.block) for t in T], dtype=torch.int32, device=self.device)
        L.select_merge_candidates(self.gdims, cands, cands.shape[0], s.budget, self.ctx_g, s.sink, s.window, s.nbr,
                                  self.idx, self.cnt, self.block[0], self.block[1] - self.block[0], self.bits,
                                  self.cap, self.ws_small, stream)
        L.sparse_decode_attn_partial(self.dims, Q, self.K, self.V, self.rows, self.bits, self.scale, self.part,
                                     self.ws_attn, stream)
        return self.part


def combine_parts(parts, out, stream=None):
    """Phase 3: out [batch][Hq][d] from the ranks' states [world][batch][Hq][d+2]."""
    L.attn_combine(parts, out, stream)


@dataclass(frozen=True)
class DecodeShape:
    batch: int
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    d_proj: int
    hidden: int            # 0: q' is supplied directly (no predictor MLP)
    inter: int
    stride: int            # producer depth stride = slots per producer call
    sink: int
    window: int
    budget: int
    nbr: int
    interval: int
    ctx_cap: int

    @property
    def n_out(self) -> int:
        return self.stride * self.n_q_heads * self.d_proj

    @property
    def idx_cap(self) -> int:
        return min((2 * self.nbr + 1) * self.budget, self.ctx_cap)

    @property
    def words(self) -> int:
        return (self.ctx_cap + 31) // 32


class SparseDecoder:
    """Owns the per-layer state of the sparse path (projected keys, predicted
    queries, selections) and the workspaces, and issues the schedule.

    K[l], V[l]: [batch][Hkv][ctx_cap][d] bf16 caches (rows of future decode
    tokens may already be present; only rows < T are ever read).
    Wk[l]: [Hkv][d'][d] bf16.  mlp[p] = (W1, W2) for each producer layer p.
    selection: "head" (one importance set per query head), "group_max" /
    "group_sum" (one set per KV head, tb_score_select_group) or "inclusive"
    (per head, at most `budget` positions after neighbour fetch,
    tb_score_select_inclusive)."""

    SELECTIONS = ("head", "group_max", "group_sum", "inclusive")

    def __init__(self, shape: DecodeShape, K, V, Wk, mlp, ctx0: list[int], steps: int, device="cuda",
                 selection: str = "head", prefetch_kv: bool = False, balance: bool = True,
                 overlap_select: bool = True, select_streams: int = 4):
        if selection not in self.SELECTIONS:
            raise ValueError(f"selection must be one of {self.SELECTIONS}")
        self.selection = selection
        # balance: after each selection, tb_attn_plan cuts the attention's
        # slices at equal shares of the kept rows, and the attention launches
        # of the interval use them (tb_sparse_decode_attn_planned).  A plan
        # costs about what one launch saves, so it pays only when several
        # launches share it: not at an interval of 1.
        self.balance = balance and shape.interval > 1
        # TB_ATTN_PREFETCH_KV for the attention launches whose preceding
        # kernel writes none of the lengths, selection words and K/V rows
        # below T-1.  Inside a step that is every attention launch except the
        # first one right after the selection of the same (only) layer; for
        # the first launch of a step the caller vouches for the kernel it ran
        # last (a K/V append of the new token's rows is fine).
        self.prefetch_kv = prefetch_kv
        s = self.shape = shape
        self.K, self.V, self.Wk, self.mlp = K, V, Wk, mlp
        self.ctx0 = list(ctx0)
        self.steps = steps
        self.device = device
        self.dims = L.dims(s.batch, s.n_q_heads, s.n_kv_heads, s.head_dim, s.d_proj, s.ctx_cap)
        self.scale = 1.0 / math.sqrt(s.head_dim)
        B, Hq, Hkv = s.batch, s.n_q_heads, s.n_kv_heads
        self.Kp = [torch.zeros(B, Hkv, s.ctx_cap, s.d_proj, dtype=torch.bfloat16, device=device)
                   for _ in range(s.n_layers)]
        self.producers = [l for l in range(s.n_layers) if l % s.stride == 0]
        self.qp = {p: torch.zeros(B, s.stride, Hq, s.d_proj, dtype=torch.float32, device=device)
                   for p in self.producers}
        self.idx = [torch.zeros(B, Hq, s.idx_cap, dtype=torch.int32, device=device) for _ in range(s.n_layers)]
        self.cnt = [torch.zeros(B, Hq, dtype=torch.int32, device=device) for _ in range(s.n_layers)]
        self.bits = [torch.zeros(B, Hq, s.words, dtype=torch.int32, device=device) for _ in range(s.n_layers)]
        self.plan = [torch.zeros(B, Hkv, L.TB_ATTN_PLAN_STRIDE, dtype=torch.int32, device=device)
                     for _ in range(s.n_layers)] if balance else None
        self.ws_sel = L.workspace(L.score_select_workspace_bytes(self.dims), device)
        self.ws_attn = L.workspace(L.attn_workspace_bytes(self.dims), device)
        self.ws_proj = L.workspace(L.project_keys_workspace_bytes(), device)
        self.ws_pred = (L.workspace(L.predict_queries_workspace_bytes(B, s.hidden, s.inter, s.n_out), device)
                        if s.hidden > 0 else None)
        # overlap_select: a prediction step's selections go round-robin over
        # the caller's stream and select_streams - 1 more (layer l to stream
        # l % select_streams, each extra stream with a selection and a plan
        # workspace of its own), so that one layer's scoring runs on the SMs
        # another layer's cluster selection leaves free.  The layers'
        # selections are independent; the attention launches wait for all.
        n_sel = max(1, int(select_streams)) if overlap_select and s.n_layers > 1 else 1
        self.overlap_select = n_sel > 1
        self.sel_lanes = [(torch.cuda.Stream(device=device),
                           L.workspace(L.score_select_workspace_bytes(self.dims), device),
                           L.workspace(L.attn_workspace_bytes(self.dims), device) if balance else None)
                          for _ in range(n_sel - 1)]
        # with the selections spread, the producers' predictor calls run on a
        # stream of their own; each selection waits only for its producer's
        self.pred_stream = torch.cuda.Stream(device=device) if self.overlap_select and s.hidden > 0 else None
        self.ctx = torch.tensor([[t + i + 1 for t in ctx0] for i in range(steps)], dtype=torch.int32,
                                device=device)
        prefill, events = projection_schedule(self.ctx0, s.window, steps)
        self.proj_events = events
        self.prefill_len = prefill
        self.proj_steps = sorted(events)
        self.proj_begin = {i: torch.tensor(events[i], dtype=torch.int32, device=device) for i in events}
        self.proj_count = {i: torch.tensor([s.window if x >= 0 else 0 for x in events[i]], dtype=torch.int32,
                                           device=device) for i in events}
        self._zero_begin = torch.zeros(B, dtype=torch.int32, device=device)
        self._prefill_t = torch.tensor(prefill, dtype=torch.int32, device=device)

    # -------------------------------------------------------------- pieces
    def prefill(self, stream=None):
        """Project the prefilled prefix [0, floor(T0/N)*N) of every layer."""
        mx = max(self.prefill_len)
        for l in range(self.shape.n_layers):
            L.project_keys(self.dims, self.K[l], self.Wk[l], self.Kp[l], self._zero_begin, self._prefill_t, mx,
                           self.ws_proj, stream)

    def project(self, step: int, layer: int, stream=None):
        if step in self.proj_begin:
            L.project_keys(self.dims, self.K[layer], self.Wk[layer], self.Kp[layer], self.proj_begin[step],
                           self.proj_count[step], self.shape.window, self.ws_proj, stream)

    def predict(self, producer: int, h, stream=None):
        W1, W2 = self.mlp[producer]
        L.predict_queries(h, W1, W2, self.qp[producer], self.ws_pred, stream)

    def workspaces(self) -> list:
        """Every workspace the decoder's launches use (for tb_workspace_check)."""
        lanes = [w for _, ws, wp in self.sel_lanes for w in (ws, wp)]
        return [w for w in [self.ws_attn, self.ws_sel, self.ws_proj, self.ws_pred] + lanes if w is not None]

    def select(self, step: int, layer: int, qp_direct=None, stream=None, ws_sel=None, ws_plan=None):
        s = self.shape
        ws_sel = self.ws_sel if ws_sel is None else ws_sel
        ws_plan = self.ws_attn if ws_plan is None else ws_plan
        if qp_direct is not None:
            qp, stride = qp_direct, s.n_q_heads * s.d_proj
        else:
            # slot j of the producer's [batch][G][Hq][d'] buffer: base + j*Hq*d',
            # batch stride G*Hq*d' (floats)
            buf = self.qp[producer_layer(layer, s.stride)]
            qp = buf.data_ptr() + query_slot(layer, s.stride) * s.n_q_heads * s.d_proj * 4
            stride = s.stride * s.n_q_heads * s.d_proj
        if self.selection == "head":
            L.score_select(self.dims, qp, stride, self.Kp[layer], self.ctx[step], s.sink, s.window, s.budget,
                           s.nbr, self.idx[layer], self.cnt[layer], self.bits[layer], ws_sel, stream)
        elif self.selection == "inclusive":
            L.score_select_inclusive(self.dims, qp, stride, self.Kp[layer], self.ctx[step], s.sink, s.window,
                                     s.budget, s.nbr, self.idx[layer], self.cnt[layer], self.bits[layer],
                                     ws_sel, stream)
        else:
            L.score_select_group(self.dims, qp, stride, self.Kp[layer], self.ctx[step], s.sink, s.window,
                                 s.budget, s.nbr, self.selection[len("group_"):], self.idx[layer],
                                 self.cnt[layer], self.bits[layer], ws_sel, stream)
        if self.balance:
            L.attn_plan(self.dims, self.bits[layer], self.ctx[step], s.sink, s.window, self.plan[layer], ws_plan,
                        stream)

    def attend(self, step: int, layer: int, Q, out, stream=None, prefetch: bool = False):
        s = self.shape
        L.attn_set_launch_mode(L.TB_ATTN_PREFETCH_KV if prefetch else L.TB_ATTN_WAIT_ALL)
        try:
            if self.balance:
                L.sparse_decode_attn_planned(self.dims, Q, self.K[layer], self.V[layer], self.ctx[step], s.sink,
                                             s.window, self.bits[layer], self.plan[layer], self.scale, out,
                                             self.ws_attn, stream)
            else:
                L.sparse_decode_attn(self.dims, Q, self.K[layer], self.V[layer], self.ctx[step], s.sink, s.window,
                                     self.bits[layer], self.scale, out, self.ws_attn, stream)
        finally:
            L.attn_set_launch_mode(L.TB_ATTN_WAIT_ALL)

    def attend_dense(self, step: int, layer: int, Q, out, stream=None, prefetch: bool = False):
        L.attn_set_launch_mode(L.TB_ATTN_PREFETCH_KV if prefetch else L.TB_ATTN_WAIT_ALL)
        try:
            L.decode_attn(self.dims, Q, self.K[layer], self.V[layer], self.ctx[step], self.scale, out,
                          self.ws_attn, stream)
        finally:
            L.attn_set_launch_mode(L.TB_ATTN_WAIT_ALL)

    # -------------------------------------------------------------- one step
    def step(self, step: int, Q, out, h=None, qp_direct=None, stream=None, marks=None, on_select=None):
        """One decode step over all layers.

        Q: [n_layers][batch][Hq][d] bf16; out: [n_layers][batch][Hq][d] fp32;
        h: [n_producers][batch][hidden] bf16 (prediction steps, MLP shapes);
        qp_direct: [n_layers][batch][Hq][d'] fp32 (shapes without an MLP).
        The selection work of a prediction step is issued before the step's
        attention launches; `marks(name)` is called between the two groups so
        a caller can bracket them with events.  `on_select(layer)`, if given,
        is called right after each layer's selection is issued (while the
        selection workspace still holds that layer's scores); the selections
        then all run on `stream`, without the extra streams."""
        s = self.shape
        if step in self.proj_begin:
            for l in range(s.n_layers):
                self.project(step, l, stream)
        if is_prediction_step(step, s.interval):
            spread = self.overlap_select and on_select is None
            ready = {}
            if spread:
                main = (torch.cuda.current_stream(self.device) if stream is None else
                        stream if isinstance(stream, torch.cuda.Stream) else torch.cuda.ExternalStream(int(stream)))
                fork = torch.cuda.Event()
                fork.record(main)
                for st in [st for st, _, _ in self.sel_lanes] + ([self.pred_stream] if self.pred_stream else []):
                    st.wait_event(fork)
            # the predictor calls first (on their own stream when spread, an
            # event after each): a layer's queries are in place before its
            # selection starts
            for l in range(s.n_layers):
                if s.hidden > 0 and l in self.qp:
                    self.predict(l, h[self.producers.index(l)], self.pred_stream if spread else stream)
                    if spread:
                        ready[l] = torch.cuda.Event()
                        ready[l].record(self.pred_stream)
            n = 1 + len(self.sel_lanes) if spread else 1
            for l in range(s.n_layers):
                qd = None if qp_direct is None else qp_direct[l]
                st, ws_sel, ws_plan = self.sel_lanes[l % n - 1] if l % n else (main if spread else stream, None, None)
                if ready:
                    st.wait_event(ready[producer_layer(l, s.stride)])
                self.select(step, l, qd, st if l % n else stream, ws_sel, ws_plan)
                if on_select:
                    on_select(l)
            if spread:
                if ready:
                    main.wait_event(ready[max(ready)])  # (the predictor stream's last call)
                for st, _, _ in self.sel_lanes:
                    join = torch.cuda.Event()
                    join.record(st)
                    main.wait_event(join)
        if marks:
            marks("attn_begin")
        # the first launch after a prediction follows the last selection the
        # caller's stream issued; when that is layer 0's own, it wrote the
        # selection words (and plan) this launch reads
        n_streams = 1 + len(self.sel_lanes) if (self.overlap_select and on_select is None) else 1
        after_own_select = (is_prediction_step(step, s.interval) and
                            main_stream_last_selected(s.n_layers, n_streams) == 0)
        for l in range(s.n_layers):
            self.attend(step, l, Q[l], out[l], stream,
                        prefetch=self.prefetch_kv and not (l == 0 and after_own_select))
        if marks:
            marks("attn_end")

    def dense_step(self, step: int, Q, out, stream=None, marks=None):
        if marks:
            marks("attn_begin")
        for l in range(self.shape.n_layers):
            self.attend_dense(step, l, Q[l], out[l], stream, prefetch=self.prefetch_kv)
        if marks:
            marks("attn_end")


# ------------------------------------------------------------------ offloaded KV

class HostBuffer:
    """Pinned host memory mapped into the device's address space, so kernels
    read and write it directly across the host link.  `dev_ptr` is the address
    to hand the library; `tensor` is a CPU tensor view of the same bytes."""

    PORTABLE, MAPPED = 1, 2

    def __init__(self, shape, dtype=torch.bfloat16):
        rt = _rt()
        self.shape, self.dtype = tuple(shape), dtype
        nbytes = math.prod(self.shape) * torch.empty(0, dtype=dtype).element_size()
        p = ctypes.c_void_p()
        err = rt.cudaHostAlloc(ctypes.byref(p), ctypes.c_size_t(nbytes), self.PORTABLE | self.MAPPED)
        if err != 0 or not p.value:
            raise RuntimeError(f"cudaHostAlloc of {nbytes} bytes failed ({err})")
        self.ptr = p.value
        dp = ctypes.c_void_p()
        err = rt.cudaHostGetDevicePointer(ctypes.byref(dp), ctypes.c_void_p(self.ptr), 0)
        if err != 0 or not dp.value:
            rt.cudaFreeHost(ctypes.c_void_p(self.ptr))
            raise RuntimeError(f"cudaHostGetDevicePointer failed ({err}): host memory is not mapped")
        self.dev_ptr = dp.value
        self._raw = (ctypes.c_uint8 * nbytes).from_address(self.ptr)
        self.tensor = torch.frombuffer(self._raw, dtype=torch.uint8).view(dtype).view(self.shape)
        self.nbytes = nbytes

    def free(self):
        if getattr(self, "ptr", None):
            self.tensor = None
            self._raw = None
            _rt().cudaFreeHost(ctypes.c_void_p(self.ptr))
            self.ptr = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def memcpy2d(dst: int, dpitch: int, src: int, spitch: int, width: int, height: int, stream) -> None:
    """cudaMemcpy2DAsync with the copy direction inferred from the addresses."""
    err = _rt().cudaMemcpy2DAsync(ctypes.c_void_p(dst), ctypes.c_size_t(dpitch), ctypes.c_void_p(src),
                                  ctypes.c_size_t(spitch), ctypes.c_size_t(width), ctypes.c_size_t(height), 4,
                                  ctypes.c_void_p(L._stream(stream)))
    if err != 0:
        raise RuntimeError(f"cudaMemcpy2DAsync failed ({err})")


class OffloadDecoder(SparseDecoder):
    """The sparse path with the KV cache in host memory: the CPU-offloading
    workload of the TokenButler summaries ("Contributions" (CPU offloading) and
    "Results" (latency at 256K+ tokens)).  The projected keys, and with them
    scoring and selection, the predictor and the queries stay on the device;
    the attention entry points are given host-mapped K and V, so only the kept
    rows cross the host link, read by the kernels themselves.  Construct with
    device K and V, project the prefill, then offload(): the caches move to
    pinned host memory and the device copies are dropped.  A batch of N new keys
    is projected from a device staging copy of its rows (the projection reads
    K through tensor maps over device memory)."""

    def offload(self):
        s = self.shape
        self.K_host, self.V_host = [], []
        for l in range(s.n_layers):
            for src, dst in ((self.K, self.K_host), (self.V, self.V_host)):
                hb = HostBuffer(src[l].shape)
                hb.tensor.copy_(src[l])
                dst.append(hb)
                src[l] = None
        self.K = [hb.dev_ptr for hb in self.K_host]
        self.V = [hb.dev_ptr for hb in self.V_host]
        torch.cuda.empty_cache()
        B, Hq, Hkv, N = s.batch, s.n_q_heads, s.n_kv_heads, s.window
        self.stage_dims = L.dims(B, Hq, Hkv, s.head_dim, s.d_proj, N)
        self.K_stage = torch.zeros(B, Hkv, N, s.head_dim, dtype=torch.bfloat16, device=self.device)
        self.Kp_stage = torch.zeros(B, Hkv, N, s.d_proj, dtype=torch.bfloat16, device=self.device)
        self.stage_begin = {i: torch.tensor([0 if x >= 0 else -1 for x in ev], dtype=torch.int32, device=self.device)
                            for i, ev in self.proj_events.items()}

    @property
    def offloaded(self) -> bool:
        return hasattr(self, "K_host")

    def project(self, step: int, layer: int, stream=None):
        if not self.offloaded:
            return super().project(step, layer, stream)
        if step not in self.proj_begin:
            return
        s = self.shape
        Hkv, N, d, dp, cap = s.n_kv_heads, s.window, s.head_dim, s.d_proj, s.ctx_cap
        begins = self.proj_events[step]
        for b, t0 in enumerate(begins):
            if t0 >= 0:   # rows [t0, t0+N) of every KV head of sequence b -> stage
                memcpy2d(self.K_stage[b].data_ptr(), N * d * 2, self.K_host[layer].ptr + (b * Hkv * cap + t0) * d * 2,
                         cap * d * 2, N * d * 2, Hkv, stream)
        L.project_keys(self.stage_dims, self.K_stage, self.Wk[layer], self.Kp_stage, self.stage_begin[step],
                       self.proj_count[step], N, self.ws_proj, stream)
        for b, t0 in enumerate(begins):
            if t0 >= 0:   # stage -> K' rows [t0, t0+N)
                memcpy2d(self.Kp[layer].data_ptr() + (b * Hkv * cap + t0) * dp * 2, cap * dp * 2,
                         self.Kp_stage[b].data_ptr(), N * dp * 2, N * dp * 2, Hkv, stream)


# ------------------------------------------------------------------ events

_cudart = None


def _rt():
    """The CUDA runtime torch already loaded (event records, pinned host
    memory, strided copies)."""
    global _cudart
    if _cudart is None:
        _cudart = ctypes.CDLL("libcudart.so.12")
        P, sz = ctypes.c_void_p, ctypes.c_size_t
        _cudart.cudaEventRecordWithFlags.argtypes = [P, P, ctypes.c_uint]
        _cudart.cudaEventRecordWithFlags.restype = ctypes.c_int
        _cudart.cudaHostAlloc.argtypes = [ctypes.POINTER(P), sz, ctypes.c_uint]
        _cudart.cudaHostAlloc.restype = ctypes.c_int
        _cudart.cudaHostGetDevicePointer.argtypes = [ctypes.POINTER(P), P, ctypes.c_uint]
        _cudart.cudaHostGetDevicePointer.restype = ctypes.c_int
        _cudart.cudaFreeHost.argtypes = [P]
        _cudart.cudaFreeHost.restype = ctypes.c_int
        _cudart.cudaMemcpy2DAsync.argtypes = [P, sz, P, sz, sz, sz, ctypes.c_int, P]
        _cudart.cudaMemcpy2DAsync.restype = ctypes.c_int
    return _cudart


def record_event(ev: torch.cuda.Event, stream: torch.cuda.Stream):
    """Record `ev` on `stream`; inside a stream capture this becomes an event
    record node of the graph (cudaEventRecordExternal), so its timestamp is
    taken on every replay."""
    err = _rt().cudaEventRecordWithFlags(ctypes.c_void_p(ev.cuda_event), ctypes.c_void_p(stream.cuda_stream), 1)
    if err != 0:
        raise RuntimeError(f"cudaEventRecordWithFlags failed ({err})")

