"""Planted mistakes: each test compiles a copy of the oracle with one plausible error (a dropped
term, a wrong sign, index or operand) into a temporary directory and requires that at least one
pin in oracle_pins.py fails against it. The real oracle is never modified."""
import os
import shutil
import subprocess
import sys

import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "bsa_oracle.c")

MUTANTS = {
    "mean_divides_by_stride": ("double mean = sum / (double)l;", "double mean = sum / (double)s;"),
    "window_starts_at_l": ("(j * s + r) * (int64_t)d", "(j * l + r) * (int64_t)d"),
    "window_drops_last_row": ("for (int r = 0; r < l; ++r) sum", "for (int r = 0; r < l - 1; ++r) sum"),
    "window_count_off_by_one": ("return (T - l) / s + 1;", "return (T - l) / s;"),
    "rounding_ties_away": ("rint(x / quantum)", "round(x / quantum)"),
    "bf16_widening_shift": ("<< 16;", "<< 15;"),
    "tau_multiplies": ("x[j] = dot / tau;", "x[j] = dot * tau;"),
    "softmax_not_normalised": ("S[j] += exp(x[j] - m) / z;", "S[j] += exp(x[j] - m);"),
    "only_first_head_scored": ("for (int h = 0; h < G; ++h) {\n        double m = -INFINITY;\n        for (int64_t j = 0; j < nc; ++j) {",
                               "for (int h = 0; h < 1; ++h) {\n        double m = -INFINITY;\n        for (int64_t j = 0; j < nc; ++j) {"),
    "overlap_touching_counts": ("end > (int64_t)block_size * b", "end >= (int64_t)block_size * b"),
    "block_min_not_max": ("if (S[j] > best) best = S[j];", "if (best == -INFINITY || S[j] < best) best = S[j];"),
    "ties_to_higher_index": ("return (a->block < b->block) ? -1 : (a->block > b->block);",
                             "return (a->block > b->block) ? -1 : (a->block < b->block);"),
    "local_window_shifted": ("int64_t local_begin = nb - n_local > 0 ? nb - n_local : 0;",
                             "int64_t local_begin = nb - n_local - 1 > 0 ? nb - n_local - 1 : 0;"),
    "boundary_wrong_candidate": ("if (take < nc) boundary[1] = cand[take].score;",
                                 "if (take < nc) boundary[1] = cand[nc - 1].score;"),
    "attention_scale_divides": ("x[i] = dot * scale;", "x[i] = dot / scale;"),
    "partial_block_drops_token": ("if (hi > T) hi = T;", "if (hi > T) hi = T - 1;"),
    "lse_drops_max": ("lse[h] = m + log(z);", "lse[h] = log(z);"),
    "head_group_interleaved": ("(int64_t)kvh * G + h) * d + c", "(int64_t)h * P->num_kv_heads + kvh) * d + c"),
    "keys_values_swapped": ("bsa_oracle_attend(qg, kp, vp,", "bsa_oracle_attend(qg, vp, kp,"),
    "forecast_drops_last_coordinate": ("for (int c = 0; c < d; ++c) dot += f[c] * ck[j * d + c];",
                                       "for (int c = 0; c < d - 1; ++c) dot += f[c] * ck[j * d + c];"),
    "forecast_vector_of_batch_row": ("bsa_oracle_load(f, P->dtype, (int64_t)pair * d + c)",
                                     "bsa_oracle_load(f, P->dtype, (int64_t)b * d + c)"),
    "forecast_scores_negated": ("        S[j] = dot;\n", "        S[j] = -dot;\n"),
}


# Child process: bind the mutant and report whether a pin fails (exit 0) or all pass (exit 1).
_CHILD = """
import sys
sys.path[:0] = [{root!r}, {tests!r}]
import oracle, oracle_pins
with oracle.using({lib!r}):
    for pin in oracle_pins.ALL_PINS:
        try:
            pin()
        except (AssertionError, ValueError) as e:
            print("caught by", pin.__name__)
            sys.exit(0)
sys.exit(1)
"""


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    find, repl = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(find) >= 1, f"mutation site for {name} not found"
    src = tmp_path / "bsa_oracle.c"
    src.write_text(text.replace(find, repl))   # every site, so the mistake is self-consistent
    shutil.copy(os.path.join(os.path.dirname(SRC), "bsa_oracle.h"), tmp_path / "bsa_oracle.h")
    lib = oracle.compile_source(str(src), str(tmp_path / f"lib_{name}.so"), str(tmp_path))
    tests = os.path.dirname(os.path.abspath(__file__))
    code = _CHILD.format(root=os.path.dirname(tests), tests=tests, lib=lib)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, f"no pin catches the planted mistake {name}: rc={r.returncode} " \
                              f"{r.stdout[-500:]} {r.stderr[-2000:]}"
