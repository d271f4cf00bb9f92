"""Plant plausible mistakes in a copy of the oracle and check that a pin catches each.

Each mutant is compiled from a textually edited copy of oracle/qsa_oracle.c into a
temporary library; the named pin test is re-run against it in a subprocess and must
fail.  Nothing here touches a GPU.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "qsa_oracle.c")

MUTANTS = {
    "tie_break_flipped": ("return (a->b < b->b) ? -1 : (a->b > b->b);",
                          "return (a->b > b->b) ? -1 : (a->b < b->b);",
                          "tests/test_oracle_invariants.py::test_constant_scores_take_lowest_blocks"),
    "query_token_dropped": ("for (int64_t j = tail0; j <= t; ++j)",
                            "for (int64_t j = tail0; j < t; ++j)",
                            "tests/test_oracle_invariants.py::test_dense_equivalence_when_budget_covers_all"),
    "head_group_interleaved": ("int g = h / GRP;", "int g = h % NKV;",
                               "tests/test_oracle_invariants.py::test_dense_equivalence_when_budget_covers_all"),
    "relu_dropped": ("double r = dot > 0.0 ? dot : 0.0;", "double r = dot;",
                     "tests/test_oracle_invariants.py::test_integer_scores_are_exact"),
    "own_block_selectable": ("int64_t n_c = t / BLK;", "int64_t n_c = (t + 1) / BLK;",
                             "tests/test_oracle_invariants.py::test_dense_equivalence_when_budget_covers_all"),
    "bf16_truncation": ("u += 0x7fffu + lsb;", "u += 0u * lsb;",
                        "tests/test_oracle_compress.py::test_rne_hand_cases"),
    "softmax_scale": ("1.0 / sqrt((double)HD)", "1.0 / (double)HD",
                      "tests/test_oracle_invariants.py::test_dense_equivalence_when_budget_covers_all"),
    "budget_off_by_one": ("for (int32_t i = 0; i < k; ++i) idx[i] = (int32_t)c[i].b;",
                          "for (int32_t i = 0; i < k; ++i) idx[i] = (int32_t)c[i + 1].b;",
                          "tests/test_oracle_invariants.py::test_monotone_scores_give_sliding_window"),
    "compress_order": ("float s012 = s01 + x2;\n                float s0123 = s012 + x3;",
                       "float s012 = s01 + x3;\n                float s0123 = s012 + x2;",
                       "tests/test_oracle_compress.py::test_order_sensitive_inputs_match_torch_fp32"),
    "score_weight_dropped": ("s += bf(w[h]) * r;", "s += r;",
                             "tests/test_oracle_brute.py::test_brute_random"),
    "kth_off_by_one": ("*kth = c[k - 1].s;", "*kth = c[k].s;",
                       "tests/test_oracle_brute.py::test_kth_is_the_boundary_score"),
    "kth_sentinel": ("*kth = -1.0;", "*kth = 0.0;",
                     "tests/test_oracle_brute.py::test_kth_is_the_boundary_score"),
    "forced_row_ignored": ("idx = (int32_t *)(forced_idx + r * topk);",
                           "idx = (int32_t *)(forced_idx);",
                           "tests/test_oracle_invariants.py::test_forced_selection_attends_exactly_the_given_blocks"),
    "forced_count_short": ("cnt = forced_cnt[r];", "cnt = forced_cnt[r] > 0 ? forced_cnt[r] - 1 : 0;",
                           "tests/test_oracle_invariants.py::test_forced_own_selection_reproduces_outputs"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pin_catches_mutant(name, tmp_path):
    old, new, pin = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                    "-o", str(so), str(mut), "-lm"], check=True)
    env = dict(os.environ, QSA_ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", pin], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pin {pin} did not catch mutant {name}:\n{r.stdout[-2000:]}"
