"""Guard regions and poisoned rows, on the GPU.

No memory checker runs on the GPUs these kernels are tested on, so stray
accesses are caught by construction instead:

* Every output, input and workspace buffer is the middle of a larger
  allocation whose head and tail guards hold a fixed bit pattern (a NaN where
  the data is floating point, a valid position where it is an index list).
  After the call both guards of every output must still hold it, and output
  entries the call does not own (index-list slots past the count, K' rows
  outside the requested range) must keep the value they were given.  A read
  past an input's end would pull a NaN or a stray position into the result.
* Every input row the method must not use holds NaN: cache rows at or past the
  sequence length, rows outside every head's attended set, K' rows outside the
  candidate range [S, T-N), K rows outside the projected range.  The result
  must still be the oracle's (attention, predictor) or identical bit for bit to
  the result on clean inputs (selection, projection).  A masked row that is
  multiplied by a zero probability still turns the output into NaN, so this
  also shows that the attention kernels never load such rows at all.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import parity
import tb_inputs
import query_aware_sparse_tb_b200 as tb

pytestmark = pytest.mark.gpu

DEV = "cuda"
GUARD_BYTES = 4096      # a multiple of 256: every view keeps its allocation's alignment
NAN32 = 0x7FC0DEAD      # a quiet fp32 NaN
NAN16 = 0x7FC1          # a quiet bf16 NaN
FILL32 = 0x5A5A5A5A
FILL8 = 0xA5
_INT = {1: torch.uint8, 2: torch.int16, 4: torch.int32}


class Guarded:
    """A contiguous device tensor of `shape` and `dtype` inside an allocation
    with a head and a tail guard of GUARD_BYTES that hold the bit pattern
    `guard`.  The tensor starts as `init` (a tensor to copy, or a bit pattern;
    by default the guard pattern)."""

    def __init__(self, shape, dtype, guard, init=None):
        es = torch.empty(0, dtype=dtype).element_size()
        self.g = GUARD_BYTES // es
        self.n = math.prod(shape)
        self.guard = guard
        self.raw = torch.full((2 * self.g + self.n,), guard, dtype=_INT[es], device=DEV)
        self.t = self.raw[self.g:self.g + self.n].view(dtype).view(shape)
        if isinstance(init, torch.Tensor):
            self.t.copy_(init)
        elif init is not None:
            self.raw[self.g:self.g + self.n] = init

    def assert_guards(self, what):
        assert torch.all(self.raw[:self.g] == self.guard), f"{what}: head guard overwritten"
        assert torch.all(self.raw[self.g + self.n:] == self.guard), f"{what}: tail guard overwritten"


def _guarded_ws(nbytes):
    """A workspace (as tb.workspace makes one) with FILL8 guards around it."""
    ws = Guarded(((nbytes + 255) // 256 * 256,), torch.uint8, FILL8)
    lib = tb._lib.load()
    tb._lib._check(lib.tb_workspace_init(ws.t.data_ptr(), ws.n, tb._lib._stream(None)))
    return ws


def _w(**kw):
    base = tb_inputs.WORKLOADS["llama8k"].scaled(name="canary", n_q_heads=8, n_kv_heads=2)
    return base.scaled(**kw)


def _dims(w):
    return tb.dims(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.d_proj, w.ctx_cap)


def _nan_rows(X, b, g, rows):
    X[b, g, rows] = float("nan")


# ----------------------------------------------------------------- attention

@pytest.mark.parametrize("d", [64, 128])
def test_dense_attention_guards_and_rows_past_length(d):
    w = _w(head_dim=d, batch=4, ctx0=2900, ctx0_lo=2900, ctx0_hi=2900, steps=4, name=f"cdense{d}")
    cap = w.ctx_cap
    ctx = [1, 37, 1500, cap]
    K, V = tb_inputs.kv_layer(w, 0, "cpu")
    for b, T in enumerate(ctx):
        for g in range(w.n_kv_heads):
            _nan_rows(K, b, g, slice(T, None))
            _nan_rows(V, b, g, slice(T, None))
    Q = tb_inputs.query(w, 0, 0, "cpu")
    Kd, Vd = Guarded(K.shape, torch.bfloat16, NAN16, K), Guarded(V.shape, torch.bfloat16, NAN16, V)
    Qd = Guarded(Q.shape, torch.bfloat16, NAN16, Q)
    dm = _dims(w)
    out = Guarded((w.batch, w.n_q_heads, d), torch.float32, NAN32)
    ws = _guarded_ws(tb.attn_workspace_bytes(dm))
    scale = 1 / math.sqrt(d)
    tb.decode_attn(dm, Qd.t, Kd.t, Vd.t, torch.tensor(ctx, dtype=torch.int32, device=DEV), scale, out.t, ws.t)
    torch.cuda.synchronize()
    assert tb.workspace_check(ws.t) == 0
    out.assert_guards("out")
    ws.assert_guards("workspace")
    Kb, Vb, Qb = parity.bits16(K), parity.bits16(V), parity.bits16(Q)
    got = out.t.cpu().numpy()
    for b in range(w.batch):
        for h in range(w.n_q_heads):
            ref = oracle.attention(Qb[b, h], Kb[b, h // 4], Vb[b, h // 4], np.arange(ctx[b], dtype=np.int32), scale)
            parity.assert_close(got[b, h], ref, f"dense b={b} h={h} T={ctx[b]}")


@pytest.mark.parametrize("d,density", [(128, 0.1), (64, 0.3)])
def test_sparse_attention_guards_and_unattended_rows(d, density):
    w = _w(head_dim=d, batch=3, ctx0=4000, ctx0_lo=4000, ctx0_hi=4000, steps=8, sink=16, window=64,
           name=f"csparse{d}")
    cap = w.ctx_cap
    ctx = [70, 2049, 4007]
    sets = tb_inputs.selection_sets(w, ctx, density)
    A = [[oracle.attention_set(ctx[b], w.sink, w.window, sets[b][h].numpy()) for h in range(w.n_q_heads)]
         for b in range(w.batch)]
    K, V = tb_inputs.kv_layer(w, 0, "cpu")
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            keep = np.zeros(cap, bool)
            for h in range(4 * g, 4 * g + 4):
                keep[A[b][h]] = True
            drop = torch.from_numpy(~keep)
            _nan_rows(K, b, g, drop)
            _nan_rows(V, b, g, drop)
    Q = tb_inputs.query(w, 1, 0, "cpu")
    Kd, Vd = Guarded(K.shape, torch.bfloat16, NAN16, K), Guarded(V.shape, torch.bfloat16, NAN16, V)
    Qd = Guarded(Q.shape, torch.bfloat16, NAN16, Q)
    W = (cap + 31) // 32
    packed = parity.pack_sets([[s.numpy() for s in hs] for hs in sets], W).view(np.int32)
    bits = Guarded(packed.shape, torch.int32, -1, torch.from_numpy(packed))
    dm = _dims(w)
    out = Guarded((w.batch, w.n_q_heads, d), torch.float32, NAN32)
    ws = _guarded_ws(tb.attn_workspace_bytes(dm))
    scale = 1 / math.sqrt(d)
    tb.sparse_decode_attn(dm, Qd.t, Kd.t, Vd.t, torch.tensor(ctx, dtype=torch.int32, device=DEV), w.sink,
                          w.window, bits.t, scale, out.t, ws.t)
    torch.cuda.synchronize()
    assert tb.workspace_check(ws.t) == 0
    out.assert_guards("out")
    ws.assert_guards("workspace")
    Kb, Vb, Qb = parity.bits16(K), parity.bits16(V), parity.bits16(Q)
    got = out.t.cpu().numpy()
    for b in range(w.batch):
        for h in range(w.n_q_heads):
            ref = oracle.attention(Qb[b, h], Kb[b, h // 4], Vb[b, h // 4], A[b][h], scale)
            parity.assert_close(got[b, h], ref, f"sparse b={b} h={h}")


# ----------------------------------------------------------------- selection

def _oracle_kp(w, K):
    Kb = parity.bits16(K)
    Wk = parity.bits16(tb_inputs.wk_layer(w, 0, "cpu"))
    Kp = np.zeros((w.batch, w.n_kv_heads, w.ctx_cap, w.d_proj), np.uint16)
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            Kp[b, g] = oracle.project_keys(Kb[b, g], Wk[g])
    return Kp


def _select(w, Kp_bits, qp, ctx, budget, nbr, sink, window, mode):
    """One guarded score+select call; returns (idx, count, bits) on the CPU
    after checking every guard and that no slot past a count was written."""
    dm = _dims(w)
    B, Hq = w.batch, w.n_q_heads
    Kp = Guarded(Kp_bits.shape, torch.bfloat16, NAN16, parity.from_bits16(Kp_bits))
    qpt = Guarded(qp.shape, torch.float32, NAN32, torch.from_numpy(np.ascontiguousarray(qp, np.float32)))
    cap = min(budget if mode == "inclusive" else (2 * nbr + 1) * budget, w.ctx_cap)
    W = (w.ctx_cap + 31) // 32
    idx = Guarded((B, Hq, cap), torch.int32, FILL32, -7)
    cnt = Guarded((B, Hq), torch.int32, FILL32, -7)
    bits = Guarded((B, Hq, W), torch.int32, FILL32, -1)
    ws = _guarded_ws(tb.score_select_workspace_bytes(dm))
    args = (dm, qpt.t, Hq * w.d_proj, Kp.t, torch.tensor(ctx, dtype=torch.int32, device=DEV), sink, window,
            budget, nbr)
    if mode == "head":
        tb.score_select(*args, idx.t, cnt.t, bits.t, ws.t)
    elif mode == "inclusive":
        tb.score_select_inclusive(*args, idx.t, cnt.t, bits.t, ws.t)
    else:
        tb.score_select_group(*args, mode, idx.t, cnt.t, bits.t, ws.t)
    torch.cuda.synchronize()
    assert tb.workspace_check(ws.t) == 0
    for buf, name in ((idx, "idx"), (cnt, "count"), (bits, "sel_bits"), (ws, "workspace")):
        buf.assert_guards(f"{mode} {name}")
    I, n = idx.t.cpu().numpy(), cnt.t.cpu().numpy()
    assert np.all((n >= 0) & (n <= cap)), mode
    for b in range(B):
        for h in range(Hq):
            assert np.all(I[b, h, n[b, h]:] == -7), f"{mode} b={b} h={h}: a slot past the count was written"
    return I, n, bits.t.cpu().numpy()


@pytest.mark.parametrize("mode", ["head", "max", "sum", "inclusive"])
def test_selection_guards_and_rows_outside_candidates(mode):
    w = _w(batch=3, ctx0=3000, ctx0_lo=3000, ctx0_hi=3000, steps=1, name=f"csel_{mode}")
    K, _ = tb_inputs.kv_layer(w, 0, "cpu")
    Kp = _oracle_kp(w, K)
    qp = tb_inputs.direct_qp(w, 0, 0, "cpu").numpy()
    ctx = [3001, 1111, 90]          # the last one takes every candidate
    budget, nbr, sink, window = 200, 1, 16, 64
    clean = _select(w, Kp, qp, ctx, budget, nbr, sink, window, mode)
    poisoned = Kp.copy()
    for b, T in enumerate(ctx):
        poisoned[b, :, :sink] = NAN16
        poisoned[b, :, max(sink, T - window):] = NAN16
    got = _select(w, poisoned, qp, ctx, budget, nbr, sink, window, mode)
    for name, x, y in zip(("idx", "count", "sel_bits"), clean, got):
        assert np.array_equal(x, y), f"{mode}: {name} depends on K' rows outside [S, T-N)"


def test_bits_from_idx_guards_and_input_bounds():
    w = _w(batch=2, ctx0=5000, ctx0_lo=5000, ctx0_hi=5000, steps=1, name="cbits")
    ctx = [5001, 999]
    sets = tb_inputs.selection_sets(w, ctx, 0.2)
    cap = 1024
    W = (w.ctx_cap + 31) // 32
    # the index list's guards hold position 5, which no set below contains:
    # reading past the list would set its bit
    host = torch.full((w.batch, w.n_q_heads, cap), 5, dtype=torch.int32)
    cnt = torch.zeros((w.batch, w.n_q_heads), dtype=torch.int32)
    want_sets = []
    for b in range(w.batch):
        row = []
        for h in range(w.n_q_heads):
            s = sets[b][h][:cap - 2]
            assert s.numel() == 0 or int(s.min()) >= w.sink > 5
            n = s.numel()
            host[b, h, :n] = s
            host[b, h, n:n + 2] = torch.tensor([-1, w.ctx_cap + 5])    # ignored entries
            cnt[b, h] = n + 2
            row.append(s.numpy())
        want_sets.append(row)
    cnt[0, 0] = cap + 10          # clamped to idx_cap: reads exactly the row
    host[0, 0, :] = torch.arange(w.sink, w.sink + cap, dtype=torch.int32)
    want_sets[0][0] = np.arange(w.sink, w.sink + cap)
    idx = Guarded(host.shape, torch.int32, 5, host)
    out = Guarded((w.batch, w.n_q_heads, W), torch.int32, FILL32, -1)
    tb.select_bits_from_idx(_dims(w), idx.t, cnt.to(DEV), out.t)
    torch.cuda.synchronize()
    out.assert_guards("sel_bits")
    assert np.array_equal(out.t.cpu().numpy().view(np.uint32), parity.pack_sets(want_sets, W))


# ----------------------------------------------------------------- projection

def test_projection_guards_and_rows_outside_range():
    w = _w(batch=2, ctx0=1000, ctx0_lo=1000, ctx0_hi=1000, steps=100, name="cproj")
    cap, dp = w.ctx_cap, w.d_proj
    K, _ = tb_inputs.kv_layer(w, 0, "cpu")
    Wk = tb_inputs.wk_layer(w, 0, DEV)
    ranges = [(37, 700), (cap - 300, 300)]      # unaligned start; a range that ends at the last row
    begin = torch.tensor([r[0] for r in ranges], dtype=torch.int32, device=DEV)
    count = torch.tensor([r[1] for r in ranges], dtype=torch.int32, device=DEV)
    poisoned = K.clone()
    for b, (lo, n) in enumerate(ranges):
        for g in range(w.n_kv_heads):
            _nan_rows(poisoned, b, g, slice(0, lo))
            _nan_rows(poisoned, b, g, slice(lo + n, None))

    def run(Kin):
        Kd = Guarded(Kin.shape, torch.bfloat16, NAN16, Kin)
        Kp = Guarded((w.batch, w.n_kv_heads, cap, dp), torch.bfloat16, NAN16, -12345)
        ws = _guarded_ws(tb.project_keys_workspace_bytes())
        tb.project_keys(_dims(w), Kd.t, Wk, Kp.t, begin, count, max(r[1] for r in ranges), ws.t)
        torch.cuda.synchronize()
        assert tb.workspace_check(ws.t) == 0
        Kp.assert_guards("K'")
        ws.assert_guards("workspace")
        return parity.bits16(Kp.t)

    clean, got = run(K), run(poisoned)
    untouched = np.uint16(np.int16(-12345).view(np.uint16))
    for b, (lo, n) in enumerate(ranges):
        assert np.all(got[b, :, :lo] == untouched) and np.all(got[b, :, lo + n:] == untouched), \
            f"b={b}: a row outside the requested range was written"
        assert np.array_equal(got[b, :, lo:lo + n], clean[b, :, lo:lo + n]), \
            f"b={b}: K' depends on K rows outside the requested range"
    parity.kprime_matches(got[1, 0, cap - 300:], parity.bits16(K)[1, 0, cap - 300:], parity.bits16(Wk)[0])


# ----------------------------------------------------------------- predictor

def test_predictor_guards():
    batch = 5
    w = tb_inputs.WORKLOADS["llama64k"].scaled(batch=batch, producer_stride=4, name="cmlp")
    W1, W2 = tb_inputs.mlp_weights(w, 0, "cpu")
    h = tb_inputs.hidden_state(w, 0, 0, "cpu")
    W1d, W2d = Guarded(W1.shape, torch.bfloat16, NAN16, W1), Guarded(W2.shape, torch.bfloat16, NAN16, W2)
    hd = Guarded(h.shape, torch.bfloat16, NAN16, h)
    qp = Guarded((batch, w.n_out), torch.float32, NAN32)
    ws = _guarded_ws(tb.predict_queries_workspace_bytes(batch, w.hidden, w.inter, w.n_out))
    tb.predict_queries(hd.t, W1d.t, W2d.t, qp.t, ws.t)
    torch.cuda.synchronize()
    assert tb.workspace_check(ws.t) == 0
    qp.assert_guards("q'")
    ws.assert_guards("workspace")
    ref = oracle.predict_queries(parity.bits16(h), parity.bits16(W1), parity.bits16(W2))
    parity.assert_close(qp.t.cpu().numpy(), ref, f"q' batch={batch}")


# ----------------------------------------------------------------- KV append

def test_kv_append_guards():
    B, Hkv, cap, nL, d = 3, 2, 300, 2, 128
    dm = tb.dims(B, 4 * Hkv, Hkv, d, 32, cap)
    g = torch.Generator(device=DEV).manual_seed(5)
    init = [torch.randn(B, Hkv, cap, d, generator=g, device=DEV).to(torch.bfloat16) for _ in range(2 * nL)]
    caches = [Guarded(c.shape, torch.bfloat16, NAN16, c) for c in init]
    src = Guarded((nL, 2, B, Hkv, d), torch.bfloat16, NAN16,
                  torch.randn(nL, 2, B, Hkv, d, generator=g, device=DEV).to(torch.bfloat16))
    ptrs = torch.tensor([c.t.data_ptr() for c in caches], dtype=torch.int64, device=DEV)
    ws = _guarded_ws(256)
    ctx = [1, 150, cap]             # the first row, a middle row, the last row of the allocation
    tb.kv_append(dm, nL, src.t, ptrs, torch.tensor(ctx, dtype=torch.int32, device=DEV), ws.t)
    torch.cuda.synchronize()
    assert tb.workspace_check(ws.t) == 0
    ws.assert_guards("workspace")
    for i, c in enumerate(caches):
        c.assert_guards(f"cache {i}")
        want = init[i].clone()
        for b in range(B):
            want[b, :, ctx[b] - 1] = src.t[i // 2, i % 2, b]
        assert torch.equal(c.t, want), f"cache {i}"
