"""Plant plausible mistakes in copies of the C oracle and check that the pins
catch every one of them (CPU only; the real oracle is never modified).

Each mutant is a textual edit of tb_oracle.c compiled into a temporary shared
library: a transposed operand, a dropped term, a flipped sign, an off-by-one
range, a reversed tie-break, a skipped rounding step.
"""
import importlib.util
import os
import shutil

import pytest

import oracle
import oracle_pins
import test_oracle_schedule

SRC = os.path.join(os.path.dirname(oracle.__file__), "tb_oracle.c")

MUTANTS = [
    ("wk_transposed", "Wk[(int64_t)j * d + i]", "Wk[(int64_t)i * dp + j]"),
    ("bf16_truncates", "double r = nearbyint(scaled);", "double r = floor(scaled);"),
    ("bf16_ties_away", "double r = nearbyint(scaled);", "double r = round(scaled);"),
    ("bf16_quantum_off", "int qexp = e - 8;", "int qexp = e - 9;"),
    ("silu_dropped", "double silu = a / (1.0 + exp(-a));", "double silu = a;"),
    ("silu_sign", "double silu = a / (1.0 + exp(-a));", "double silu = a / (1.0 + exp(a));"),
    ("w1_transposed", "W1[(int64_t)i * hidden + k]", "W1[(int64_t)k * inter + i]"),
    ("score_sign", "acc += (double)qp[j] * orc_bf16_to_double(Kp[t * dp + j]);",
     "acc -= (double)qp[j] * orc_bf16_to_double(Kp[t * dp + j]);"),
    ("score_drops_last_dim", "for (int j = 0; j < dp; ++j)\n            acc += (double)qp[j]",
     "for (int j = 0; j < dp - 1; ++j)\n            acc += (double)qp[j]"),
    ("tie_break_reversed", "return (x->t < y->t) ? -1 : (x->t > y->t) ? 1 : 0;",
     "return (x->t > y->t) ? -1 : (x->t < y->t) ? 1 : 0;"),
    ("ascending_scores", "if (x->s > y->s) return -1;\n    if (x->s < y->s) return 1;",
     "if (x->s < y->s) return -1;\n    if (x->s > y->s) return 1;"),
    ("neighbour_right_dropped", "for (int64_t u = t - r; u <= t + r; ++u)",
     "for (int64_t u = t - r; u < t + r; ++u)"),
    ("candidates_into_window", "int64_t c_lo = S, c_hi = T - N;", "int64_t c_lo = S, c_hi = T - N + 1;"),
    ("candidates_into_sink", "int64_t c_lo = S, c_hi = T - N;", "int64_t c_lo = S - 1, c_hi = T - N;"),
    ("budget_off_by_one", "int64_t take = B < nC ? B : nC;", "int64_t take = B - 1 < nC ? B - 1 : nC;"),
    ("window_short", "int64_t win_begin = T - N > S ? T - N : S;",
     "int64_t win_begin = T - N + 1 > S ? T - N + 1 : S;"),
    ("sink_dropped", "for (int64_t t = 0; t < sink_end; ++t) A[n++] = (int32_t)t;", ""),
    ("scale_dropped", "z[k] = acc * scale;", "z[k] = acc;"),
    ("softmax_unnormalised", "out[j] = (float)(o / l);", "out[j] = (float)o;"),
    ("v_row_misindexed", "V[(int64_t)A[k] * d + j]", "V[(int64_t)k * d + j]"),
    ("group_max_is_min", "g = sh > g ? sh : g;", "g = sh < g ? sh : g;"),
    ("group_drops_last_head", "for (int h = 0; h < G; ++h) {", "for (int h = 0; h < G - 1; ++h) {"),
    ("group_sum_in_double", "        float g = 0.0f;", "        double g = 0.0;"),
    ("inclusive_allows_overshoot", "if (size + fresh > B) break;", "if (size + fresh > B + 1) break;"),
    ("inclusive_skips_instead_of_stopping", "if (size + fresh > B) break;", "if (size + fresh > B) continue;"),
    ("inclusive_counts_covered", "fresh += !in_set[u - lo];", "fresh += 1;"),
    ("projection_drops_last_input", "for (int i = 0; i < d; ++i)\n                acc += orc_bf16_to_double(K[",
     "for (int i = 0; i < d - 1; ++i)\n                acc += orc_bf16_to_double(K["),
    ("w2_transposed", "W2[(int64_t)o * inter + i]", "W2[(int64_t)i * n_out + o]"),
    ("predict_ignores_batch", "h[(int64_t)b * hidden + k]", "h[k]"),
    ("activation_not_rounded", [
        ("uint16_t *act = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)inter);",
         "double *act = (double *)malloc(sizeof(double) * (size_t)inter);"),
        ("act[i] = orc_double_to_bf16(silu);", "act[i] = silu;"),
        ("q += orc_bf16_to_double(act[i]) *", "q += act[i] *"),
    ], None),
    ("neighbour_left_dropped", "for (int64_t u = t - r; u <= t + r; ++u)",
     "for (int64_t u = t - r + 1; u <= t + r; ++u)"),
    ("window_long", "int64_t win_begin = T - N > S ? T - N : S;",
     "int64_t win_begin = T - N - 1 > S ? T - N - 1 : S;"),
    ("softmax_no_max_shift", "z[k] = exp(z[k] - zmax);", "z[k] = exp(z[k]);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(name, old, new, tmp_path):
    # one (old, new) edit, or a list of edits that make one mistake together
    edits = old if isinstance(old, list) else [(old, new)]
    src = open(SRC).read()
    for o, n in edits:
        assert src.count(o) == 1, f"mutation site for {name} not unique/found: {o!r}"
        src = src.replace(o, n)
    mut_src = tmp_path / "tb_oracle_mut.c"
    mut_src.write_text(src)
    so = oracle.build(force=True, src=str(mut_src), out=str(tmp_path / "libmut.so"))
    lib = oracle.load(so)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
            break
    assert caught, f"no pin caught mutant {name}"
    shutil.rmtree(tmp_path, ignore_errors=True)


# The decode-loop schedule (oracle/schedule.py): mutated copies are loaded as
# a module of the oracle package and must fail one of the schedule tests.
SCHEDULE_SRC = os.path.join(os.path.dirname(oracle.__file__), "schedule.py")

SCHEDULE_MUTANTS = [
    ("prediction_every_step", "    return step % interval == 0", "    return True"),
    ("prefix_not_whole_batches", "    proj = (ctx0 // window) * window\n", "    proj = ctx0\n"),
    ("slot_ignored", "qp = qp_cache[(k, p)][:, slot_of(layer, w.producer_stride)]", "qp = qp_cache[(k, p)][:, 0]"),
    ("selection_length_off_by_one", "T = ctx0[b] + i + 1\n                    hi = T - w.window",
     "T = ctx0[b] + i\n                    hi = T - w.window"),
    ("window_frozen_at_prediction", "T = ctx0[b] + i + 1\n                    for h in heads:",
     "T = ctx0[b] + last_prediction_step(i, w.interval) + 1\n                    for h in heads:"),
]

SCHEDULE_CHECKS = [getattr(test_oracle_schedule, n) for n in dir(test_oracle_schedule)
                   if n.startswith("test_") and callable(getattr(test_oracle_schedule, n))]


def _load_schedule(text, tmp_path):
    path = tmp_path / "schedule_mut.py"
    path.write_text(text)
    spec = importlib.util.spec_from_file_location("oracle.schedule_mut", str(path))
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name,old,new", SCHEDULE_MUTANTS, ids=[m[0] for m in SCHEDULE_MUTANTS])
def test_schedule_checks_catch_mutant(name, old, new, tmp_path, monkeypatch):
    src = open(SCHEDULE_SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique/found"
    monkeypatch.setattr(test_oracle_schedule, "schedule", _load_schedule(src.replace(old, new), tmp_path))
    caught = []
    for check in SCHEDULE_CHECKS:
        try:
            check()
        except (AssertionError, ValueError, IndexError):
            caught.append(check.__name__)
            break
    assert caught, f"no schedule check caught mutant {name}"
