"""Helpers for the GPU parity tests: conversions between torch tensors and the
oracle's numpy arrays, bit packing of index sets, and the comparison rules.

Tolerances (bf16 inputs, fp32 accumulation and fp32 softmax on the GPU; the
oracle sums in double):
  attention output   max |gpu - oracle| <= 2e-3 and ||gpu - oracle|| / ||oracle|| <= 1e-3
  predicted queries  the same two bounds
  projected keys     bit-exact, except an element whose exact value lies within
                     the fp32 accumulation error bound eps = 2 n 2^-24 sum|k w|
                     of a bf16 rounding midpoint: there any bf16 value within
                     eps + one spacing of the exact value is a correct result
                     of "fp32 accumulate, then round to bf16"
  selected sets      bit-exact on integer-valued inputs; otherwise they may
                     differ only within +-nbr of a candidate whose oracle score
                     is within 1e-4 * max(1, |s_B|) of the B-th score s_B
"""
from __future__ import annotations

import numpy as np
import torch

MAX_ABS = 2e-3
REL_L2 = 1e-3
SCORE_TIE_TOL = 1e-4


def bits16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def from_bits16(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def bf16_to_f64(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def pack_sets(sets, W: int) -> np.ndarray:
    """Index sets [b][h] -> uint32 bitmap [B][Hq][W] (bit t%32 of word t/32)."""
    B, Hq = len(sets), len(sets[0])
    out = np.zeros((B, Hq, W), np.uint32)
    for b in range(B):
        for h in range(Hq):
            t = np.asarray(sets[b][h], np.int64)
            if t.size:
                np.bitwise_or.at(out[b, h], t >> 5, (np.uint32(1) << (t & 31).astype(np.uint32)))
    return out


def assert_close(gpu: np.ndarray, ref: np.ndarray, what: str, max_abs=MAX_ABS, rel_l2=REL_L2):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU values"
    err = np.abs(gpu - ref)
    rel = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err.max() <= max_abs, f"{what}: max abs err {err.max():.3e} > {max_abs}"
    assert rel <= rel_l2, f"{what}: rel L2 err {rel:.3e} > {rel_l2}"


def kprime_matches(gpu_bits: np.ndarray, K_bits: np.ndarray, W_bits: np.ndarray):
    """Check projected keys against the exact product: each element must be the
    bf16 rounding of the exact value, except where the exact value is within
    the fp32 accumulation bound of a rounding midpoint (then either neighbour
    is accepted).  Returns (n_ambiguous, n_total)."""
    K = bf16_to_f64(K_bits)
    W = bf16_to_f64(W_bits)
    exact = K @ W.T
    absum = np.abs(K) @ np.abs(W).T
    n = K.shape[1]
    eps = 2.0 * n * 2.0 ** -24 * absum          # generous fp32 summation bound
    g = bf16_to_f64(gpu_bits)
    # bf16 spacing around |exact|: 2^(floor(log2|x|) - 7)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.maximum(np.abs(exact), 1e-38)))
    ulp = 2.0 ** (e - 7)
    down = np.floor(exact / ulp) * ulp
    mid = down + ulp / 2
    ambiguous = np.abs(exact - mid) <= eps
    # the fp32 sum f is within eps of the exact value and g is f rounded to
    # bf16, so |g - exact| <= eps + half a spacing; when the sum nearly cancels,
    # eps can exceed the spacing of the tiny result and g may sit several
    # spacings away
    near = np.abs(g - exact) <= eps + ulp * (1 + 1e-9)
    # unambiguous elements: the correctly rounded value (within half a spacing,
    # and strictly closer than the neighbour)
    correct = np.abs(g - exact) <= ulp / 2 * (1 + 1e-12)
    ok = np.where(ambiguous, near, correct)
    bad = np.argwhere(~ok)
    assert bad.size == 0, f"K' mismatch at {bad[:5].tolist()}: gpu {g[tuple(bad[0])]} exact {exact[tuple(bad[0])]}"
    return int(ambiguous.sum()), int(exact.size)


def assert_sets_match(gpu_set, ref_set, ref_scores, lo: int, budget: int, nbr: int, exact: bool, what: str):
    """Compare a GPU selected set with the oracle's.  ref_scores[k] is the
    oracle's fp32 score of candidate lo + k."""
    g = np.asarray(gpu_set, np.int64)
    r = np.asarray(ref_set, np.int64)
    assert np.all(np.diff(g) > 0), f"{what}: GPU set not sorted/unique"
    if exact:
        assert np.array_equal(g, r), f"{what}: sets differ: gpu-only {np.setdiff1d(g, r)[:8]}, " \
                                     f"oracle-only {np.setdiff1d(r, g)[:8]}"
        return 0
    diff = np.setxor1d(g, r)
    if diff.size == 0:
        return 0
    s = np.asarray(ref_scores, np.float64)
    order = np.lexsort((np.arange(s.size), -s))
    sB = s[order[min(budget, s.size) - 1]]
    tol = SCORE_TIE_TOL * max(1.0, abs(sB))
    exempt = np.nonzero(np.abs(s - sB) <= tol)[0] + lo
    for t in diff:
        assert np.any(np.abs(exempt - t) <= nbr), \
            f"{what}: position {t} differs and is not within {nbr} of a near-tie candidate (s_B={sB})"
    return int(diff.size)


# ----------------------------------------------------------------------------
# Exact validity of a selection against the scores it was taken from.
#
# The GPU's fp32 scores can differ from the oracle's in the last bits (another
# summation order), so on random inputs the two sets may differ at near-ties.
# These checks close that gap without feeding anything the GPU produced into
# the oracle: (1) the GPU's own scores (tb_score_select_scores) must lie within
# the fp32 summation bound of the oracle's scores of the same inputs, and (2)
# the GPU's set must be exactly the set the selection rule gives on the GPU's
# own scores.  (2) is a restatement of the rule for checking only (test side,
# numpy); the oracle itself never sees GPU data.
# ----------------------------------------------------------------------------

def f32_sum_bound(q: np.ndarray, Kp_bits: np.ndarray) -> np.ndarray:
    """Largest |fp32 sequential sum - exact sum| plus the oracle's one rounding
    to fp32, for the scores q . K'[t] (q float [d'], K' bf16 bits [n][d'])."""
    kf = bf16_to_f64(Kp_bits)
    absum = np.abs(kf) @ np.abs(np.asarray(q, np.float64))
    return (kf.shape[1] + 2) * 2.0 ** -24 * absum


def assert_scores_within(gpu: np.ndarray, ref: np.ndarray, bound: np.ndarray, what: str):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU scores"
    err = np.abs(gpu - ref)
    bad = np.nonzero(err > bound + 1e-30)[0]
    assert bad.size == 0, f"{what}: score {bad[0]} off by {err[bad[0]]:.3e} > bound {bound[bad[0]]:.3e}"


def rule_topb(scores: np.ndarray, lo: int, budget: int, nbr: int) -> np.ndarray:
    """Top-`budget` of the candidates lo, lo+1, ... by (score desc, position
    asc), expanded by +-nbr and clipped to the candidate range; sorted."""
    s = np.asarray(scores, np.float32)
    n = s.size
    if n == 0:
        return np.zeros(0, np.int64)
    order = np.lexsort((np.arange(n), -s.astype(np.float64)))
    keep = np.zeros(n, bool)
    top = order[:min(budget, n)]
    for k in range(-nbr, nbr + 1):
        j = top + k
        keep[j[(j >= 0) & (j < n)]] = True
    return np.nonzero(keep)[0] + lo


def rule_inclusive(scores: np.ndarray, lo: int, budget: int, nbr: int) -> np.ndarray:
    """Candidates in (score desc, position asc) order while the union of their
    +-nbr neighbourhoods, clipped to the candidate range, holds at most
    `budget` positions; the union, sorted."""
    s = np.asarray(scores, np.float32)
    n = s.size
    covered = np.zeros(n, bool)
    used = 0
    for t in np.lexsort((np.arange(n), -s.astype(np.float64))):
        a, b = max(0, t - nbr), min(n, t + nbr + 1)
        new = int((~covered[a:b]).sum())
        if used + new > budget:
            break
        covered[a:b] = True
        used += new
    return np.nonzero(covered)[0] + lo


def assert_selection_valid(gpu_set, gpu_scores, lo: int, budget: int, nbr: int, what: str,
                           inclusive: bool = False):
    """The GPU set must be exactly what the rule gives on the GPU's own fp32
    scores of the candidates lo, lo+1, ..."""
    want = (rule_inclusive if inclusive else rule_topb)(gpu_scores, lo, budget, nbr)
    g = np.asarray(gpu_set, np.int64)
    assert np.array_equal(g, want), f"{what}: not the rule's set on the kernel's own scores: " \
                                    f"gpu-only {np.setdiff1d(g, want)[:8]}, rule-only {np.setdiff1d(want, g)[:8]}"
