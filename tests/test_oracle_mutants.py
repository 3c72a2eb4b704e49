"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a private copy of the oracle's C source (on
the CPU, never in the product), builds it, and runs the pin suite against
the broken build: the suite must fail.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "hkv_oracle.c")

MUTANTS = {
    "window_not_strict": ("*label = (uint8_t)(need < W ? 1 : 0);",
                          "*label = (uint8_t)(need <= W ? 1 : 0);"),
    "accumulate_from_oldest": ("c += p_row[n - 1 - delta];", "c += p_row[delta];"),
    "reach_is_strict": ("if (c >= tau) {", "if (c > tau) {"),
    "near_excludes_D": ("if (stratified && delta <= D) nearv[nn++] = e;",
                        "if (stratified && delta < D) nearv[nn++] = e;"),
    "current_token_candidate": ("if (delta < 1) continue;  /* only past tokens are candidates */",
                                "if (delta < 0) continue;"),
    "tie_keeps_lower_pos": ("return (x->pos > y->pos) - (x->pos < y->pos);",
                            "return (x->pos < y->pos) - (x->pos > y->pos);"),
    "budget_rounds_up": ("*budget_g = ng > 0 ? (int32_t)((T - (int64_t)nl * W) / ng) : 0;",
                         "*budget_g = ng > 0 ? (int32_t)((T - (int64_t)nl * W + ng - 1) / ng) : 0;"),
    "scale_by_d": ("const double scale = 1.0 / sqrt((double)d);",
                   "const double scale = 1.0 / (double)d;"),
    "score_window_off_by_one": ("for (int32_t step = t - r + 1; step <= t; ++step) {",
                                "for (int32_t step = t - r; step <= t; ++step) {"),
    "local_window_too_wide": ("if (S->kept[i] > t - W) S->kept[w++] = S->kept[i];",
                              "if (S->kept[i] >= t - W) S->kept[w++] = S->kept[i];"),
    "evict_highest": ("if (x->s < y->s) return -1;\n    if (x->s > y->s) return 1;",
                      "if (x->s < y->s) return 1;\n    if (x->s > y->s) return -1;"),
    "no_causal_mask": ("int32_t nvis = pos + 1 < n_k ? pos + 1 : n_k;",
                       "int32_t nvis = n_k;"),
    "class_row_by_position": ("for (int32_t delta = 0; delta <= i; ++delta) row[P - 1 - delta] += wi[i - delta];",
                              "for (int32_t delta = 0; delta <= i; ++delta) row[i - delta] += wi[i - delta];"),
    "class_row_mean_over_P": ("for (int32_t j = 0; j < P; ++j) row[j] /= (double)nq;",
                              "for (int32_t j = 0; j < P; ++j) row[j] /= (double)P;"),
    "select_band_absolute": ("else if (max_gone > min_kept * (1.0 + band)) ok = 0;",
                             "else if (max_gone - min_kept > band) ok = 0;"),
    "select_band_wrong_side": ("else if (max_gone > min_kept * (1.0 + band)) ok = 0;",
                               "else if (max_gone > min_kept * (1.0 - band)) ok = 0;"),
    "label_band_one_sided": ("if (fabs(out->c_window[h] - prm->tau) <= prm->label_band) {",
                             "if (out->c_window[h] - prm->tau <= prm->label_band) {"),
    "ste_scores_ignore_step_cache": ("if (kept[i] <= step) { rows[nv] = kept[i]; where[nv] = i; ++nv; }",
                                     "{ rows[nv] = kept[i]; where[nv] = i; ++nv; }"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mdir = tmp_path / "oracle"
    mdir.mkdir()
    (mdir / "hkv_oracle.c").write_text(src.replace(old, new))
    (mdir / "hkv_oracle.h").write_text(open(os.path.join(ROOT, "oracle", "hkv_oracle.h")).read())
    so = mdir / "libhkv_oracle.so"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-std=c11", "-shared", "-fPIC",
                           "-o", str(so), str(mdir / "hkv_oracle.c"), "-lm"])
    env = dict(os.environ, HKV_ORACLE_SO=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch mutant {name}:\n{r.stdout[-2000:]}"
