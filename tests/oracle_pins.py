"""Checks that pin the oracle to something other than itself.

Each ``pin_*`` function takes a loaded oracle library and raises AssertionError
on a mismatch.  They are run against the real oracle by test_oracle_pins.py and
against deliberately broken copies of it by test_oracle_mutants.py, which checks
that every planted mistake is caught by at least one pin.

What pins what:
  bf16 rounding      torch's float32 -> bf16 conversion (a library routine) on
                     random, midpoint and subnormal values, plus closed-form
                     cases where rounding through float32 first would differ
  key projection     exact integer matrix products (numpy int64) rounded by torch
  predictor MLP      torch float64 matmul + SiLU as an independent witness
  scores             exact integer dot products (numpy int64)
  group scores       exact integer closed forms (max over heads, dot product
                     with the summed queries), a case where fp32 head-order
                     rounding decides the sum, and the invariant that identical
                     heads select what one head selects
  selection          hand-worked golden cases, and brute force by rank counting
                     on tiny inputs with many ties
  inclusive budget   a hand-worked case, brute force (the union recomputed from
                     scratch for every prefix of the score order), and r = 0,
                     where it is the plain top-B
  attention set      sink/window/importance invariants
  attention          closed forms (two-logit softmax, equal logits, constant V),
                     torch float64 softmax as a witness, sparse == dense when the
                     budget covers every candidate
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def _bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()


def _round_f64_via_torch(x: np.ndarray) -> np.ndarray:
    """Round exactly-representable-in-float32 doubles to bf16 with torch."""
    f = np.asarray(x, np.float64).astype(np.float32)
    assert np.all(f.astype(np.float64) == x), "witness needs float32-exact inputs"
    return _bf16_bits(torch.from_numpy(f))


# ---------------------------------------------------------------------------
# bf16 rounding
# ---------------------------------------------------------------------------

def pin_bf16_rounding(lib):
    rng = np.random.default_rng(1)
    vals = [rng.standard_normal(4000).astype(np.float32),
            (rng.standard_normal(2000) * 1e-39).astype(np.float32),   # subnormal range
            (rng.standard_normal(2000) * 1e30).astype(np.float32)]
    # exact midpoints between adjacent bf16 values (ties go to the even code)
    base = rng.integers(0x0080, 0x7f00, 2000).astype(np.uint32)
    mids = ((base << 16) | 0x8000).view(np.float32)
    vals.append(mids)
    vals.append(-mids)
    x = np.concatenate(vals).astype(np.float64)
    got = np.array([lib.orc_double_to_bf16(float(v)) for v in x], np.uint16)
    want = _round_f64_via_torch(x)
    assert np.array_equal(got, want), "bf16 rounding disagrees with torch"
    # a double just above a bf16 midpoint must round up; rounding to float32 first
    # would land on the midpoint and then round to even (down)
    one_up = lib.orc_double_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -40)
    assert one_up == 0x3F81, hex(one_up)
    assert lib.orc_double_to_bf16(1.0 + 2.0 ** -8) == 0x3F80          # tie -> even
    assert lib.orc_double_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82      # tie -> even (up)
    assert lib.orc_double_to_bf16(-2.5) == 0xC020
    assert lib.orc_double_to_bf16(1e39) == 0x7F80                     # overflow -> inf


def pin_bf16_widening(lib):
    bits = np.arange(0, 1 << 16, 7, dtype=np.uint32).astype(np.uint16)
    finite = (bits & 0x7F80) != 0x7F80
    bits = bits[finite]
    got = np.array([lib.orc_bf16_to_double(int(b)) for b in bits])
    want = _bits_to_f64(bits)
    assert np.array_equal(got, want)


# ---------------------------------------------------------------------------
# key projection
# ---------------------------------------------------------------------------

def pin_project_keys_integer(lib):
    rng = np.random.default_rng(2)
    for (rows, d, dp) in [(37, 64, 16), (5, 128, 32), (1, 8, 16)]:
        K = rng.integers(-4, 5, (rows, d))
        W = rng.integers(-4, 5, (dp, d))
        exact = K.astype(np.int64) @ W.astype(np.int64).T          # [rows][dp]
        want = _round_f64_via_torch(exact.astype(np.float64))
        got = oracle.project_keys(_bf16_bits(torch.tensor(K, dtype=torch.float32)),
                                  _bf16_bits(torch.tensor(W, dtype=torch.float32)), lib=lib)
        assert np.array_equal(got, want), (rows, d, dp)


def pin_project_keys_random(lib):
    g = torch.Generator().manual_seed(3)
    K = torch.randn(64, 128, generator=g).bfloat16()
    W = (torch.randn(32, 128, generator=g) * 0.02).bfloat16()
    got = _bits_to_f64(oracle.project_keys(_bf16_bits(K), _bf16_bits(W), lib=lib))
    ref = (K.double() @ W.double().T).numpy()
    # one bf16 rounding (8 significant bits) of the exact product: relative
    # error at most the unit roundoff 2^-8
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 * (1 + 1e-12) + 1e-300)
    # and the nearest code: the adjacent bf16 codes are not closer
    bits = oracle.project_keys(_bf16_bits(K), _bf16_bits(W), lib=lib).astype(np.int32)
    for step in (-1, 1):
        nb = _bits_to_f64((bits + step).astype(np.uint16))
        assert np.all(np.abs(nb - ref) >= np.abs(got - ref))
    assert np.mean(got == ref) < 0.5, "inputs are not trivially exact"


# ---------------------------------------------------------------------------
# predictor MLP
# ---------------------------------------------------------------------------

def pin_predict_queries(lib):
    g = torch.Generator().manual_seed(4)
    B, hidden, inter, n_out = 3, 256, 96, 40
    h = torch.randn(B, hidden, generator=g).bfloat16()
    W1 = (torch.randn(inter, hidden, generator=g) * 0.1).bfloat16()
    W2 = (torch.randn(n_out, inter, generator=g) * 0.1).bfloat16()
    got = oracle.predict_queries(_bf16_bits(h), _bf16_bits(W1), _bf16_bits(W2), lib=lib)
    a = h.double() @ W1.double().T
    act = torch.nn.functional.silu(a).bfloat16().double()
    want = (act @ W2.double().T).numpy()
    # the witness rounds the activation through float32; rare double-rounding
    # cases move one activation by one bf16 step, far inside this bound
    err = np.abs(got.astype(np.float64) - want)
    assert np.all(err <= 1e-3 * np.abs(want).max() + 1e-6), err.max()
    # h = 0 gives SiLU(0) = 0 and q' = 0 exactly
    z = oracle.predict_queries(_bf16_bits(torch.zeros(1, hidden)), _bf16_bits(W1),
                               _bf16_bits(W2), lib=lib)
    assert np.all(z == 0.0)


def _bf16_rne(x: float) -> float:
    """Round a double to the nearest bf16 value, ties to even (normal range)."""
    if x == 0.0:
        return 0.0
    quantum = 2.0 ** (math.floor(math.log2(abs(x))) - 7)
    return round(x / quantum) * quantum          # x / quantum is exact; round() ties to even


def pin_predict_queries_silu_closed_form(lib):
    # hidden 1, W1 = identity row, W2 = identity: q' = bf16_rne(SiLU(h)) exactly
    # (reading R6: the activation is rounded to bf16 before the second product).
    # Each SiLU value here lies at least 0.1 bf16 spacings from a rounding
    # midpoint and is not itself a bf16 value, so the rounding is visible.
    xs = [-2.0, 0.5, 3.0, -0.75, 5.5]
    hvals = torch.tensor([[x] for x in xs])
    W1 = torch.ones(1, 1)
    W2 = torch.ones(1, 1)
    got = oracle.predict_queries(_bf16_bits(hvals), _bf16_bits(W1), _bf16_bits(W2), lib=lib)
    for k, x in enumerate(xs):
        silu = x / (1.0 + math.exp(-x))
        want = _bf16_rne(silu)
        assert want != silu
        assert float(got[k, 0]) == want, (x, float(got[k, 0]), want)


# ---------------------------------------------------------------------------
# scores
# ---------------------------------------------------------------------------

def pin_scores_integer(lib):
    rng = np.random.default_rng(5)
    for dp in (16, 32):
        Kp = rng.integers(-300, 301, (50, dp))
        q = rng.integers(-4, 5, dp)
        Kp_bits = _bf16_bits(torch.tensor(Kp, dtype=torch.float32))
        Kp_val = _bits_to_f64(Kp_bits).astype(np.int64)               # bf16 codes of Kp
        want = (Kp_val @ q.astype(np.int64)).astype(np.float64)
        got = oracle.scores(q.astype(np.float32), Kp_bits, 7, 50, lib=lib)
        assert np.array_equal(got.astype(np.float64), want[7:50])


def pin_group_scores_integer(lib):
    rng = np.random.default_rng(11)
    for dp in (16, 32):
        Kp = rng.integers(-300, 301, (60, dp))
        q = rng.integers(-4, 5, (4, dp))
        Kp_bits = _bf16_bits(torch.tensor(Kp, dtype=torch.float32))
        Kp_val = _bits_to_f64(Kp_bits).astype(np.int64)
        per_head = Kp_val @ q.T.astype(np.int64)                           # [60][4], exact
        got = oracle.group_scores(q.astype(np.float32), Kp_bits, 5, 60, "max", lib=lib)
        assert np.array_equal(got.astype(np.float64), per_head.max(axis=1)[5:].astype(np.float64))
        # |sum| <= 4 * 4 * 300 * 32 < 2^24: every fp32 partial sum is exact
        got = oracle.group_scores(q.astype(np.float32), Kp_bits, 5, 60, "sum", lib=lib)
        assert np.array_equal(got.astype(np.float64), (Kp_val @ q.sum(axis=0))[5:].astype(np.float64))


def pin_group_sum_fp32_head_order(lib):
    # head scores 2^24, 1, 1, 0 at one position.  In fp32, in head order, each
    # "+ 1" is a tie that rounds to the even 2^24, so the group sum is 2^24;
    # in the reverse order 1 + 1 = 2 first, and 2^24 + 2 is representable.
    Kp_bits = _bf16_bits(torch.tensor([[1.0] + [0.0] * 15], dtype=torch.float32))
    q = np.zeros((4, 16), np.float32)
    q[0, 0], q[1, 0], q[2, 0] = 2.0 ** 24, 1.0, 1.0
    assert oracle.group_scores(q, Kp_bits, 0, 1, "sum", lib=lib)[0] == np.float32(2.0 ** 24)
    assert oracle.group_scores(q[::-1].copy(), Kp_bits, 0, 1, "sum", lib=lib)[0] == np.float32(2.0 ** 24 + 2)
    assert oracle.group_scores(q, Kp_bits, 0, 1, "max", lib=lib)[0] == np.float32(2.0 ** 24)


def pin_group_selection_identical_heads(lib):
    rng = np.random.default_rng(12)
    T, S, N, B, r = 120, 4, 8, 17, 1
    Kp_bits = _bf16_bits(torch.randn(T, 16, generator=torch.Generator().manual_seed(12)))
    q1 = rng.standard_normal(16).astype(np.float32)
    per_head = oracle.select(oracle.scores(q1, Kp_bits, S, T - N, lib=lib), T, S, N, B, r, lib=lib)
    for red in ("max", "sum"):
        s = oracle.group_scores(np.stack([q1] * 4), Kp_bits, S, T - N, red, lib=lib)
        assert oracle.select(s, T, S, N, B, r, lib=lib).tolist() == per_head.tolist(), red


# ---------------------------------------------------------------------------
# selection
# ---------------------------------------------------------------------------

def pin_select_golden(lib):
    with open(os.path.join(GOLDEN, "select_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        got = oracle.select(np.array(c["scores"], np.float32), c["T"], c["S"], c["N"], c["B"],
                            c["r"], lib=lib)
        assert got.tolist() == c["expect"], (c["name"], got.tolist())


def _brute_select(s, T, S, N, B, r):
    lo, hi = S, T - N
    C = list(range(lo, hi))
    top = []
    for t in C:
        rank = sum(1 for u in C if s[u - lo] > s[t - lo] or (s[u - lo] == s[t - lo] and u < t))
        if rank < B:
            top.append(t)
    keep = set()
    for t in top:
        for u in range(t - r, t + r + 1):
            if lo <= u < hi:
                keep.add(u)
    return sorted(keep)


def pin_select_brute_force(lib):
    rng = np.random.default_rng(6)
    for trial in range(300):
        S = int(rng.integers(0, 5))
        N = int(rng.integers(1, 6))
        T = int(rng.integers(1, 40))
        B = int(rng.integers(1, 12))
        r = int(rng.integers(0, 3))
        nC = max(0, T - N - S)
        s = rng.integers(-3, 4, nC).astype(np.float32)        # many ties
        if trial % 3 == 0:
            s = rng.standard_normal(nC).astype(np.float32)
        got = oracle.select(s, T, S, N, B, r, lib=lib).tolist()
        want = _brute_select(s, T, S, N, B, r)
        assert got == want, (S, N, T, B, r, s.tolist(), got, want)


def pin_select_inclusive_worked_case(lib):
    # C = [10, 15), scores fall with position, B = 4, r = 1: t=10 brings {10, 11}
    # (9 is the sink), 11 brings 12, 12 brings 13, and 13 would make 5 > 4.
    s = np.array([5, 4, 3, 2, 1], np.float32)
    assert oracle.select_inclusive(s, 20, 10, 5, 4, 1, lib=lib).tolist() == [10, 11, 12, 13]
    # C = [0, 6), B = 5, r = 1, order 0, 2, 1, 3, 4, 5: t=0 brings {0, 1}, t=2
    # brings {2, 3}, t=1 is already covered and costs nothing, t=3 brings 4,
    # and t=4 would bring 5 (6 > 5).  Stopping at the free candidate would
    # give [0, 1, 2, 3].
    s = np.array([9, 6, 8, 1, 1, 1], np.float32)
    assert oracle.select_inclusive(s, 6, 0, 0, 5, 1, lib=lib).tolist() == [0, 1, 2, 3, 4]


def _brute_select_inclusive(s, T, S, N, B, r):
    lo, hi = S, T - N
    order = sorted(range(lo, hi), key=lambda t: (-float(s[t - lo]), t))
    best = []
    for k in range(len(order) + 1):
        union = sorted({u for t in order[:k] for u in range(t - r, t + r + 1) if lo <= u < hi})
        if len(union) > B:
            break
        best = union
    return best


def pin_select_inclusive_brute_force(lib):
    rng = np.random.default_rng(13)
    for trial in range(300):
        S = int(rng.integers(0, 5))
        N = int(rng.integers(1, 6))
        T = int(rng.integers(1, 40))
        B = int(rng.integers(1, 14))
        r = int(rng.integers(0, 3))
        nC = max(0, T - N - S)
        s = rng.integers(-3, 4, nC).astype(np.float32)
        if trial % 3 == 0:
            s = rng.standard_normal(nC).astype(np.float32)
        got = oracle.select_inclusive(s, T, S, N, B, r, lib=lib).tolist()
        assert got == _brute_select_inclusive(s, T, S, N, B, r), (S, N, T, B, r, s.tolist(), got)
        if r == 0:
            assert got == oracle.select(s, T, S, N, B, 0, lib=lib).tolist()


# ---------------------------------------------------------------------------
# attention set and attention
# ---------------------------------------------------------------------------

def pin_attention_set(lib):
    rng = np.random.default_rng(7)
    for _ in range(200):
        S = int(rng.integers(0, 6))
        N = int(rng.integers(1, 8))
        T = int(rng.integers(1, 60))
        lo, hi = S, T - N
        I = np.array(sorted(x for x in range(lo, hi) if rng.random() < 0.3), np.int32)
        A = oracle.attention_set(T, S, N, I, lib=lib).tolist()
        sink = set(range(0, min(S, T)))
        window = set(range(max(S, T - N), T))
        assert A == sorted(set(A)), "sorted and unique"
        assert set(A) == sink | window | set(I.tolist())
        if T <= S + N:
            assert A == list(range(T)), "short context is dense"


def pin_attention_golden(lib):
    with open(os.path.join(GOLDEN, "attention_cases.json")) as f:
        cases = {c["name"]: c for c in json.load(f)["cases"]}

    def run(c):
        q = _bf16_bits(torch.tensor(c["q"], dtype=torch.float32))
        K = _bf16_bits(torch.tensor(c["K"], dtype=torch.float32))
        V = _bf16_bits(torch.tensor(c["V"], dtype=torch.float32))
        return oracle.attention(q, K, V, np.array(c["rows"], np.int32), c["scale"], lib=lib)

    e2 = math.exp(2.0)
    o = run(cases["two_rows"])
    assert np.allclose(o, [1 / (1 + e2), e2 / (1 + e2)], rtol=1e-7, atol=0)
    o = run(cases["two_rows_scaled"])
    assert np.allclose(o, [(4 * e2) / (1 + e2), (-2 * e2 + 2) / (1 + e2)], rtol=1e-7, atol=0)
    o = run(cases["row_subset"])
    assert np.allclose(o, [2.0, 3.0], rtol=1e-7, atol=0)
    em16 = math.exp(-16.0)
    o = run(cases["large_logits"])
    assert np.allclose(o, [1 / (1 + em16), em16 / (1 + em16)], rtol=1e-7, atol=0)


def pin_attention_constant_v(lib):
    g = torch.Generator().manual_seed(8)
    d, rows = 64, 40
    q = _bf16_bits(torch.randn(d, generator=g))
    K = _bf16_bits(torch.randn(rows, d, generator=g) * 3)
    v = torch.randn(d, generator=g).bfloat16()
    V = _bf16_bits(v.float().expand(rows, d).contiguous())
    A = np.array([0, 3, 5, 17, 39], np.int32)
    o = oracle.attention(q, K, V, A, 0.125, lib=lib)
    assert np.allclose(o, v.float().numpy(), rtol=1e-6, atol=0)


def pin_attention_torch_witness(lib):
    g = torch.Generator().manual_seed(9)
    d, rows = 128, 300
    q = torch.randn(d, generator=g).bfloat16()
    K = torch.randn(rows, d, generator=g).bfloat16()
    V = torch.randn(rows, d, generator=g).bfloat16()
    A = np.array(sorted(set(np.random.default_rng(9).integers(0, rows, 120).tolist())), np.int32)
    scale = 1 / math.sqrt(d)
    got = oracle.attention(_bf16_bits(q), _bf16_bits(K), _bf16_bits(V), A, scale, lib=lib)
    Ks, Vs = K.double()[torch.from_numpy(A).long()], V.double()[torch.from_numpy(A).long()]
    p = torch.softmax((Ks @ q.double()) * scale, dim=0)
    want = (p @ Vs).numpy()
    assert np.allclose(got, want, rtol=1e-6, atol=1e-7)


def pin_sparse_equals_dense_when_budget_covers(lib):
    g = torch.Generator().manual_seed(10)
    T, S, N, d, dp = 90, 4, 8, 64, 16
    K = torch.randn(T, d, generator=g).bfloat16()
    V = torch.randn(T, d, generator=g).bfloat16()
    W = (torch.randn(dp, d, generator=g) * 0.1).bfloat16()
    q = torch.randn(d, generator=g).bfloat16()
    qp = torch.randn(dp, generator=g).numpy().astype(np.float32)
    Kp = oracle.project_keys(_bf16_bits(K), _bf16_bits(W), lib=lib)
    s = oracle.scores(qp, Kp, S, T - N, lib=lib)
    I = oracle.select(s, T, S, N, T, 1, lib=lib)                    # budget >= |C|
    A = oracle.attention_set(T, S, N, I, lib=lib)
    assert A.tolist() == list(range(T))
    sparse = oracle.attention(_bf16_bits(q), _bf16_bits(K), _bf16_bits(V), A, 0.125, lib=lib)
    p = torch.softmax((K.double() @ q.double()) * 0.125, dim=0)
    dense = (p @ V.double()).numpy()
    assert np.allclose(sparse, dense, rtol=1e-6, atol=1e-7)


ALL_PINS = [
    pin_bf16_rounding,
    pin_bf16_widening,
    pin_project_keys_integer,
    pin_project_keys_random,
    pin_predict_queries,
    pin_predict_queries_silu_closed_form,
    pin_scores_integer,
    pin_group_scores_integer,
    pin_group_sum_fp32_head_order,
    pin_group_selection_identical_heads,
    pin_select_golden,
    pin_select_brute_force,
    pin_select_inclusive_worked_case,
    pin_select_inclusive_brute_force,
    pin_attention_set,
    pin_attention_golden,
    pin_attention_constant_v,
    pin_attention_torch_witness,
    pin_sparse_equals_dense_when_budget_covers,
]
