"""The oracle's pins catch plausible mistakes: each test plants one mistake
in a copy of the oracle (on the CPU), and the pin suite must fail on it.

The C oracle is copied with one line changed, compiled with the same flags,
and the pins run against it in a child pytest (TSO_MUTANT_LIB points the
oracle's loader at the mutated build).  The n-gram oracle is Python: its
mutants replace one function in-process.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ts_oracle.c")

# name -> (the correct line, the planted mistake)
C_MUTANTS = {
    "path_without_self": ("for (int a = node; a >= 0; a = parent[a])",
                          "for (int a = parent[node]; a >= 0; a = parent[a])"),
    "wrong_gqa_head_map": ("const int g = h / group;", "const int g = h % n_heads_kv;"),
    "penalty_sign_swapped": ("x = x > 0.0f ? x / penalty : x * penalty;",
                             "x = x > 0.0f ? x * penalty : x / penalty;"),
    "importance_without_1_over_G": ("sc[n] += s[n] / z / (double)group;",
                                    "sc[n] += s[n] / z;"),
    "validity_ignores_parent": ("valid[i] = valid[p] && tokens[i] == argmax[p];",
                                "valid[i] = tokens[i] == argmax[p];"),
    "argmax_ties_to_highest_id": ("if (x > best) {", "if (x >= best) {"),
    "select_ties_to_higher_position": ("return (x->pos > y->pos) - (x->pos < y->pos);",
                                       "return (x->pos < y->pos) - (x->pos > y->pos);"),
    "accept_ties_to_highest_index": ("if (valid[i] && depth[i] > depth[best])",
                                     "if (valid[i] && depth[i] >= depth[best])"),
    "path_window_includes_root": ("for (int a = i; a != 0; a = parent[a])",
                                  "for (int a = i; a >= 0; a = parent[a])"),
    "path_window_without_self": ("for (int a = i; a != 0; a = parent[a])",
                                 "for (int a = parent[i]; a > 0; a = parent[a])"),
    "random_tie_off_by_one": ("int pick = (int)(r % (uint64_t)count), best = 0;",
                              "int pick = (int)((r + 1) % (uint64_t)count), best = 0;"),
    "path_penalty_sign_swapped": ("x = (x > 0.0f) ? (x / penalty) : (x * penalty);",
                                  "x = (x > 0.0f) ? (x * penalty) : (x / penalty);"),
    "path_argmax_ties_to_highest_id": ("if (best < x) {", "if (best <= x) {"),
    "random_tie_validity_ignores_parent": ("valid[i] = tokens[i] == argmax[p] && valid[p];",
                                           "valid[i] = tokens[i] == argmax[p];"),
    "sample_multiplies_by_temperature": ("float z = penalized[at] / temperature;",
                                         "float z = penalized[at] * temperature;"),
    "sample_ignores_noise": ("z = z + gumbel[at];", "z = z + 0.0f;"),
    "sample_subtracts_noise": ("z = z + gumbel[at];", "z = z - gumbel[at];"),
    "sample_ties_to_highest_id": ("if (best < z) {", "if (best <= z) {"),
    "commit_writes_rows_in_place": (
        "memcpy(base + ((int64_t)n_ctx + j) * head_dim, rows + (size_t)j * head_dim,",
        "memcpy(base + ((int64_t)n_ctx + accept[2 + j]) * head_dim, rows + (size_t)j * head_dim,"),
}


def _pins_with(src_text, tmp_path):
    """Compile `src_text` as the oracle and run the pin suite against it;
    returns the child pytest's exit code (0 all passed, 1 some failed)."""
    mut = tmp_path / "ts_oracle.c"
    mut.write_text(src_text)
    lib = tmp_path / "libts_oracle_mutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                           "-fno-fast-math", "-ffp-contract=off", str(mut), "-o", str(lib),
                           "-lm"])
    env = dict(os.environ, TSO_MUTANT_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:]


def test_unchanged_oracle_copy_passes_the_pins(tmp_path):
    # the control: the same route with nothing planted passes
    code, out = _pins_with(open(SRC).read(), tmp_path)
    assert code == 0, out


@pytest.mark.parametrize("name", sorted(C_MUTANTS))
def test_pins_catch_planted_c_oracle_mistake(name, tmp_path):
    good, bad = C_MUTANTS[name]
    src = open(SRC).read()
    assert src.count(good) == 1, f"{name}: the line to change must be unique"
    code, out = _pins_with(src.replace(good, bad), tmp_path)
    assert code == 1, f"{name}: the pins did not catch it\n{out}"


# ------------------------------------------------------- n-gram oracle
def _update_off_by_one(counts, text, n_new, n):
    out = dict(counts)
    for e in range(max(n - 1, len(text) - n_new + 1), len(text)):   # misses the first new end
        g = tuple(int(x) for x in text[e - n + 1:e + 1])
        out[g] = out.get(g, 0) + 1
    return out


def _topk_ties_descending(counts, first, k):
    cands = [(g[1:], c) for g, c in counts.items() if g[0] == first]
    cands.sort(key=lambda gc: (-gc[1], tuple(-x for x in gc[0])))
    return cands[:k]


def _counts_drop_last_window(text, n):
    counts = {}
    for i in range(len(text) - n):   # one window short
        g = tuple(int(x) for x in text[i:i + n])
        counts[g] = counts.get(g, 0) + 1
    return counts


@pytest.mark.parametrize("name,fn,mutant", [
    ("update_off_by_one", "ngram_update", _update_off_by_one),
    ("topk_ties_descending", "ngram_topk", _topk_ties_descending),
    ("counts_drop_last_window", "ngram_counts", _counts_drop_last_window),
])
def test_pins_catch_planted_ngram_oracle_mistake(name, fn, mutant, monkeypatch):
    import test_ngram as T
    from oracle import ngram as O
    monkeypatch.setattr(O, fn, mutant)
    pins = [T.test_oracle_hand_counted_alternation, T.test_oracle_distinct_tokens_count_once,
            T.test_oracle_golden_figure_example,
            T.test_oracle_update_counts_only_windows_ending_in_the_new_tokens,
            T.test_oracle_topk_order_breaks_ties_by_continuation,
            lambda: T.test_oracle_periodic_text_closed_form(5, 31, 4)]
    failed = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed >= 1, f"{name}: no pin failed"
