"""The test-side restatements of the selection rules (tests/parity.py), which
the GPU tests use to check a selection against the kernel's own scores, agree
with the oracle's selection on random tiny inputs with many ties.  This pins
the checker to the pinned oracle, so a mistake in either shows here."""
import numpy as np
import pytest

import oracle
import parity


@pytest.mark.parametrize("inclusive", [False, True])
def test_rules_match_the_oracle(inclusive):
    rng = np.random.default_rng(7)
    for case in range(400):
        S = int(rng.integers(0, 6))
        N = int(rng.integers(1, 8))
        T = int(rng.integers(1, 90))
        B = int(rng.integers(1, 30))
        r = int(rng.integers(0, 4))
        n = max(0, T - N - S)
        # coarse values: many exact ties, negative and positive zeros
        s = (rng.integers(-3, 4, n) * rng.choice([1.0, 0.5], n)).astype(np.float32)
        s[rng.random(n) < 0.1] = -0.0
        if inclusive:
            want = oracle.select_inclusive(s, T, S, N, B, r)
            got = parity.rule_inclusive(s, S, B, r)
        else:
            want = oracle.select(s, T, S, N, B, r)
            got = parity.rule_topb(s, S, B, r)
        assert np.array_equal(got, want), (case, S, N, T, B, r)


def test_score_bound_catches_a_wrong_score():
    rng = np.random.default_rng(3)
    q = rng.standard_normal(32).astype(np.float32)
    Kp = oracle.project_keys(rng.integers(0, 1 << 16, (50, 128)).astype(np.uint16) & np.uint16(0xBFFF),
                             rng.integers(0, 1 << 16, (32, 128)).astype(np.uint16) & np.uint16(0x3FFF))
    s = oracle.scores(q, Kp, 0, 50)
    bound = parity.f32_sum_bound(q, Kp)
    parity.assert_scores_within(s, s, bound, "identical")
    bad = s.copy()
    bad[7] = np.float32(bad[7] + 4 * bound[7] + 1e-6)
    with pytest.raises(AssertionError):
        parity.assert_scores_within(bad, s, bound, "perturbed")


def test_validity_check_catches_a_wrong_set():
    s = np.array([5, 1, 3, 3, 0, 2], np.float32)
    # top-2 of candidates 10..15 by (score desc, position asc): 10 (5), 12 (3); +-1: 10, 11, 12, 13
    parity.assert_selection_valid(np.array([10, 11, 12, 13]), s, 10, 2, 1, "ok")
    with pytest.raises(AssertionError):
        parity.assert_selection_valid(np.array([10, 11, 13, 14]), s, 10, 2, 1, "tie to the higher position")
