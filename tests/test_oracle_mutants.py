"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the C oracle (on the CPU: a flipped
sign, an off-by-one window, a dropped term, a swapped operand, ...), builds
it, and checks that at least one pin of tests/test_oracle_pins.py fails on
it, while the unmodified oracle passes them all."""
import ctypes
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins
import test_oracle_scoring as scoring
import test_oracle_importance as importance
import test_oracle_ffn as ffn

SRC = os.path.join(os.path.dirname(oracle.__file__), "rk_oracle.c")

MUTANTS = {
    "rope_sign": ("y[m] = x0 * c - x1 * s;", "y[m] = x0 * c + x1 * s;"),
    "rope_pair_index": ("double x0 = x[m], x1 = x[m + h];", "double x0 = x[m], x1 = x[h - 1 - m];"),
    "window_off_by_one": ("return j > i - t->window;", "return j >= i - t->window;"),
    "causal_excludes_diagonal": ("j >= t->L || j > i) return 0;", "j >= t->L || j >= i) return 0;"),
    "retrieval_ignores_list": ("return t->uncached[j] || t->in_s[j / t->pr->p];", "return t->uncached[j];"),
    "delta_sign": ("int delta = sg[1] - sg[3];", "int delta = sg[3] - sg[1];"),
    "relocated_k_sin_sign": ("kj[m] = x0 * cs[m] - x1 * cs[h + m];", "kj[m] = x0 * cs[m] + x1 * cs[h + m];"),
    "value_is_key": ("const double* vj = aj->vr + (size_t)j * d;", "const double* vj = aj->kr + (size_t)j * d;"),
    "no_normalisation": ("for (int c = 0; c < d; ++c) o[c] /= sum;", ";"),
    "lse_drops_max": ("aj->lse[idx] = mx + log(sum);", "aj->lse[idx] = log(sum);"),
    "n_valid_always_p": ("int nv = L - k * P < P ? L - k * P : P;", "int nv = P;"),
    "page_offset": ("int page_in_seg = (k * P - sg[1]) / P;", "int page_in_seg = (k * P - sg[1]) / P + 1;"),
    # retrieval page scoring
    "score_no_relocation": ("ora_rope_rotate(x, d, theta, (double)shift, kr);",
                            "ora_rope_rotate(x, d, theta, 0.0, kr);"),
    "score_shift_sign": ("ora_rope_rotate(x, d, theta, (double)shift, kr);",
                         "ora_rope_rotate(x, d, theta, -(double)shift, kr);"),
    "score_rows_summed": ("u[c] += acc / n_rows;", "u[c] += acc;"),
    "score_one_head": ("for (int hh = kvh * g; hh < kvh * g + g; ++hh) {",
                       "for (int hh = kvh * g; hh < kvh * g + 1; ++hh) {"),
    "score_ties_upper": ("if (best < 0 || scores_out[pg] > scores_out[best]) best = pg;",
                         "if (best < 0 || scores_out[pg] >= scores_out[best]) best = pg;"),
    "score_uncached_candidates": ("if (t.uncached[j0] || j0 > last_row) continue;",
                                  "if (j0 > last_row) continue;"),
    # attention importance
    "importance_unnormalised": ("if (s[j] > -INFINITY) imp_out[j] += exp(s[j] - lse);",
                                "if (s[j] > -INFINITY) imp_out[j] += exp(s[j] - mx);"),
    "importance_wrong_head": ("int h = kvh * g + hg;", "int h = hg;"),
    "importance_shift_sign": ("int dpos = sg[1] - sg[3];", "int dpos = sg[3] - sg[1];"),
    "importance_sin_sign": ("kj[m] = x0 * cos(a) - x1 * sin(a);",
                            "kj[m] = x0 * cos(a) + x1 * sin(a);"),
    "importance_unscaled": ("s[j] = acc * scale;\n          if (s[j] > mx) mx = s[j];\n        }\n        if (mx == -INFINITY) continue;",
                            "s[j] = acc;\n          if (s[j] > mx) mx = s[j];\n        }\n        if (mx == -INFINITY) continue;"),
    # token-selective FFN
    "ffn_gate_up_swapped": ("h[f] = g / (1.0 + exp(-g)) * u;", "h[f] = u / (1.0 + exp(-u)) * g;"),
    "ffn_no_residual": ("y[n] = xd[n] + acc;", "y[n] = acc;"),
    "ffn_relu": ("h[f] = g / (1.0 + exp(-g)) * u;", "h[f] = (g > 0.0 ? g : 0.0) * u;"),
    "ffn_sigmoid_sign": ("h[f] = g / (1.0 + exp(-g)) * u;", "h[f] = g / (1.0 + exp(g)) * u;"),
    "ffn_down_transposed": ("const uint16_t* wdr = j->wd + (size_t)n * df;\n    double acc = 0.0;\n    for (int f = 0; f < df; ++f) acc += h[f] * bf16_to_double(wdr[f]);",
                            "double acc = 0.0;\n    for (int f = 0; f < df; ++f) acc += h[f] * bf16_to_double(j->wd[(size_t)f * dm + n % dm]);"),
}

PIN_CALLS = [
    lambda: [pins.test_rope_matches_complex_rotation(d) for d in (4, 64)],
    pins.test_rope_quarter_turn_by_hand,
    pins.test_global_head_is_causal_attention,
    pins.test_local_head_is_sliding_window,
    pins.test_retrieval_head_is_union_mask,
    pins.test_cfg1_page_table_by_hand,
    pins.test_partial_last_page_by_hand,
    lambda: [pins.test_visible_pairs_brute_force("cfg1")],
    scoring.test_scores_equal_bilinear_expansion,
    scoring.test_planted_pages_win,
    scoring.test_few_candidates_all_picked_and_other_tables_empty,
    scoring.test_ties_go_to_the_lower_page,
    importance.test_importance_is_dense_softmax_column_sums_cfg1,
    importance.test_importance_is_dense_softmax_column_sums_retrieval,
    importance.test_zero_keys_give_harmonic_sums,
    ffn.test_one_feature_by_hand,
    ffn.test_two_features_by_hand,
    ffn.test_mirrored_features_give_a_bilinear_form,
    ffn.test_zero_gate_is_the_residual_path,
    ffn.test_down_projection_scales_the_update_and_rows_follow_the_list,
]


def _build(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, name
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / f"{name}.so"
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-D_DEFAULT_SOURCE", "-shared", "-fPIC",
                           "-pthread", "-o", str(so), str(path), "-lm"])
    return str(so)


def _fails_some_pin(so_path, monkeypatch):
    monkeypatch.setattr(oracle, "_lib", None)
    monkeypatch.setattr(oracle, "build", lambda force=False: so_path)
    for call in PIN_CALLS:
        try:
            call()
        except AssertionError:
            return True
    return False


def test_unmodified_oracle_passes(tmp_path, monkeypatch):
    so = _build(tmp_path, "clean", "#include <math.h>", "#include <math.h>")
    assert not _fails_some_pin(so, monkeypatch)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, monkeypatch, name):
    old, new = MUTANTS[name]
    so = _build(tmp_path, name, old, new)
    assert _fails_some_pin(so, monkeypatch), f"no pin catches mutant {name}"
