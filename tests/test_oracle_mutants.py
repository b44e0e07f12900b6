"""The pins have teeth: plant plausible mistakes in copies of the oracle source
(compiled on the CPU into a temporary library) and check that each one makes
at least one pin fail.  The real oracle is untouched."""
import ctypes
import inspect
import os
import subprocess

import numpy as np
import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "rotate forward instead of back": ("const double kx = xt * ca + yt * sa;\n    const double ky = -xt * sa + yt * ca;",
                                       "const double kx = xt * ca - yt * sa;\n    const double ky = xt * sa + yt * ca;"),
    "distance sign": ("cur + (double)p->offsets[j] - kpos", "kpos - cur - (double)p->offsets[j]"),
    "sum instead of mean over offsets": ("s_trig += acc / (double)p->n_offsets;", "s_trig += acc;"),
    "phase difference sign": ("cos(w * dist + c_arg - k_arg)", "cos(w * dist - c_arg + k_arg)"),
    "norm weight R instead of 1-R": ("(1.0 - p->mrl[o])", "(p->mrl[o])"),
    "frequency exponent": ("pow(theta, -2.0 * (double)f / (double)D)", "pow(theta, -(double)f / (double)D)"),
    "half-split pairing": ("*yi = f + D / 2;", "*yi = f + 1;"),
    "sample std": ("var /= (double)(T > 0 ? T : 1);", "var /= (double)(T > 1 ? T - 1 : 1);"),
    "group sum instead of max": ("if (zt > sc[t]) sc[t] = zt;", "sc[t] = (j == 0 ? 0.0 : sc[t]) + zt;"),
    "ties to the higher slot": ("return (x->slot > y->slot) - (x->slot < y->slot);",
                                "return (x->slot < y->slot) - (x->slot > y->slot);"),
    "keep the lowest scores": ("if (x->score > y->score) return -1;\n  if (x->score < y->score) return 1;",
                               "if (x->score < y->score) return -1;\n  if (x->score > y->score) return 1;"),
    "gather off by one": ("const int64_t src = base + s[j];", "const int64_t src = base + s[j] + (j > 0);"),
    "MRL from the sum of norms": ("hypot(centre[2 * o], centre[2 * o + 1]) / mean_norm[o]",
                                  "hypot(centre[2 * o], centre[2 * o + 1]) / (mean_norm[o] * (double)N)"),
    "conjugated centre": ("const double cx = p->centre[2 * o], cy = p->centre[2 * o + 1];",
                          "const double cx = p->centre[2 * o], cy = -p->centre[2 * o + 1];"),
    "head budget ignored": ("const int32_t keep = unit_budget(p, l, g);",
                            "const int32_t keep = p->budget;"),
    "unit length ignored": ("return p->unit_len ? p->unit_len[((int64_t)l * p->Hkv + g) * p->B + b] : p->seq_len[b];",
                            "return p->seq_len[b];"),
    "kept count one short of the head budget": (
        "unit_len_out[u] = (int32_t)(T < kept_max ? T : kept_max);",
        "unit_len_out[u] = (int32_t)(T < kept_max ? T : kept_max - 1);"),
}

PIN_TESTS = [
    (pins.test_worked_example_closed_form, {}),
    (pins.test_calibration_identical_queries_concentrate_fully, {}),
    (pins.test_calibration_antipodal_and_two_directions, {}),
    (pins.test_offset_mean_matches_dirichlet_closed_form, {"layout": 0}),
    (pins.test_zero_spread_equals_mean_post_rope_logit, {"layout": 0}),
    (pins.test_diffuse_queries_reduce_to_weighted_key_norm, {}),
    (pins.test_key_position_cancels, {}),
    (pins.test_zscore_invariants_and_max, {}),
    (pins.test_select_equals_brute_force_with_ties, {"T": 64, "budget": 7}),
    (pins.test_compaction_moves_selected_rows_in_order, {}),
    (pins.test_uniform_head_budgets_are_the_plain_prune, {}),
    (pins.test_head_budgets_keep_each_heads_top_b, {}),
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name!r} not found exactly once"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", str(path), "-o",
                    str(lib), "-lm"], check=True)
    real = oracle.lib()
    mutant = ctypes.CDLL(str(lib))
    for fn in ("orc_calibrate", "orc_key_score", "orc_raw_scores", "orc_zmax", "orc_select",
               "orc_compact"):
        getattr(mutant, fn).argtypes = getattr(real, fn).argtypes
        getattr(mutant, fn).restype = getattr(real, fn).restype
    caught = []
    oracle._lib = mutant
    try:
        for test, kw in PIN_TESTS:
            try:
                test(**kw)
            except AssertionError:
                caught.append(test.__name__)
    finally:
        oracle._lib = real
    assert caught, f"no pin caught the planted mistake {name!r}"


# Mistakes in the decode-loop steps of the oracle (Python functions of the package).
PY_MUTANTS = {
    "window threshold off by one": ("prune_window", "if T >= thr or T <= bud:",
                                    "if T > thr or T <= bud:"),
    "window ignored": ("prune_window", "thr = bud + max(int(window), 1)", "thr = bud + 1"),
    "appended position not advanced": ("append", "pos[l, g, slot] = cur_pos[b] + 1",
                                       "pos[l, g, slot] = cur_pos[b]"),
    "append over the newest token": ("append", "slot = int(seq_start[b]) + T",
                                     "slot = int(seq_start[b]) + max(T - 1, 0)"),
    "full segment overwritten": ("append", "if (Ts < 0).any() or (Ts >= room).any():",
                                 "if (Ts < 0).any() or (Ts > room).any():"),
    "softmax without the max shift": ("decode_attention", "w = np.exp(logits - logits.max())",
                                      "w = np.exp(logits)"),
    "KV head by modulo": ("decode_attention", "g = h // G", "g = h % Hkv"),
    "logit scale ignored": ("decode_attention", "logits = scale * (K @ qf[b, h])",
                            "logits = K @ qf[b, h]"),
    "weights not normalised": ("decode_attention", "out[b, h] = (w / w.sum()) @ V",
                               "out[b, h] = w @ V"),
    "one key short": ("decode_attention", "K = f64(k[layer, g, s0:s0 + T])",
                      "K = f64(k[layer, g, s0:s0 + T - 1])"),
}

PY_PIN_TESTS = [pins.test_prune_window_threshold,
                pins.test_head_budget_window_decides_per_unit,
                pins.test_append_and_attention_follow_each_units_length,
                pins.test_append_writes_the_next_slot_and_advances,
                pins.test_decode_loop_lengths_follow_the_window_sawtooth,
                pins.test_attention_single_key_returns_its_value,
                pins.test_attention_two_keys_closed_form,
                pins.test_attention_equal_keys_average_the_values,
                pins.test_attention_query_heads_read_their_own_kv_head,
                pins.test_attention_ignores_slot_order_and_empty_sequences,
                pins.test_attention_large_logits_pick_the_best_key]


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_planted_decode_loop_mistake_is_caught(name, monkeypatch):
    fn, old, new = PY_MUTANTS[name]
    src = inspect.getsource(getattr(oracle, fn))
    assert src.count(old) == 1, f"mutation site for {name!r} not found exactly once"
    ns = dict(vars(oracle))
    exec(src.replace(old, new), ns)
    monkeypatch.setattr(oracle, fn, ns[fn])
    caught = []
    for test in PY_PIN_TESTS:
        try:
            with np.errstate(all="ignore"):  # a mutant may overflow on purpose
                test()
        except Exception:  # a failed assertion, or the mutant indexing out of its arrays
            caught.append(test.__name__)
    assert caught, f"no pin caught the planted mistake {name!r}"
