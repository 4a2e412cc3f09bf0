"""The oracle's pins must be sharp: plant plausible slips in copies of the
oracle source (CPU only), rebuild each copy, and check that the pin suite
rejects every one of them.

Each mutant changes one thing a careless transcription could get wrong: a
dropped factor, a flipped sign, an off-by-one neighbour, a boundary rule on
the wrong step or the wrong precedence between terminated and truncated.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from oracle import oracle as oracle_mod

from . import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle_mod.__file__), "rlscan_oracle.c")

MUTANTS = {
    "gae_drop_gamma_in_carry": ("gamma * lambda * next_adv", "lambda * next_adv"),
    "gae_value_sign": ("double delta = (double)r[t] + gamma * next_v - (double)v[t];",
                       "double delta = (double)r[t] + gamma * next_v + (double)v[t];"),
    "truncation_ignored": ("if (trunc_row && trunc_row[t]) return (double)tv_row[t];",
                           "if (trunc_row && trunc_row[t]) return 0.0;"),
    "truncation_wins_over_termination": (
        "  if (term_row[t]) return 0.0;\n  if (trunc_row && trunc_row[t]) return (double)tv_row[t];",
        "  if (trunc_row && trunc_row[t]) return (double)tv_row[t];\n  if (term_row[t]) return 0.0;"),
    "window_end_drops_bootstrap": ("return bootstrap ? (double)bootstrap[n] : 0.0;", "return 0.0;"),
    "td_lambda_weights_swapped": ("((1.0 - lambda) * (double)v[t + 1] + lambda * next_g)",
                                  "(lambda * (double)v[t + 1] + (1.0 - lambda) * next_g)"),
    "vtrace_c_uses_rho_bar": ("double c = lambda * dmin(c_bar, ratio);",
                              "double c = lambda * dmin(rho_bar, ratio);"),
    "vtrace_pg_uses_value_not_vs": ("succ_vs = next_vs;", "succ_vs = (double)v[t + 1];"),
    "retrace_trace_at_wrong_step": (
        "gamma * (next_e - next_c * next_q + next_c * next_qret)",
        "gamma * (next_e - c * next_q + c * next_qret)"),
    "retrace_q_transposed": ("double qa = (double)qrow[a];", "double qa = (double)prow[a];"),
    "elig_reset_on_same_step": ("if (t > 0 && (te[t - 1] || (tr && tr[t - 1]))) prev = 0.0;",
                                "if (te[t] || (tr && tr[t])) prev = 0.0;"),
    "prefix_ignores_truncation": ("if (t > 0 && (te[t - 1] || (tr && tr[t - 1]))) s = 0;",
                                  "if (t > 0 && te[t - 1]) s = 0;"),
    "affine_reset_ignored": ("if (!(reset && reset[i])) v += (double)a[i] * carry;",
                             "v += (double)a[i] * carry;"),
    "affine_init_ignored": ("double carry = init ? (double)init[n] : 0.0;", "double carry = 0.0;"),
    "affine_grad_reset_ignored": ("if (have_next && !reset_next) g += a_next * g_next;",
                                  "if (have_next) g += a_next * g_next;"),
    "affine_grad_wrong_neighbour": ("xp = (double)x[n * T + (reverse ? t + 1 : t - 1)];",
                                    "xp = (double)x[n * T + (reverse ? t - 1 : t + 1)];"),
    "affine_tm_row_major_index": ("const int64_t i = t * N + n;", "const int64_t i = n * T + t;"),
    "affine_tm_ignores_direction": ("const int64_t t = reverse ? T - 1 - k : k;\n      const int64_t i = t * N + n;",
                                    "const int64_t t = k;\n      const int64_t i = t * N + n;"),
}

PIN_TESTS = [
    lambda: pins.test_gae_matches_bruteforce_sum(),
    lambda: pins.test_discounted_matches_bruteforce_sum(),
    lambda: pins.test_td_lambda_matches_nstep_average(),
    lambda: pins.test_vtrace_matches_impala_sum(0.95, 1.0, 0.9),
    lambda: pins.test_vtrace_matches_impala_sum(0.7, 2.0, 1.5),
    lambda: pins.test_retrace_matches_munos_sum(3),
    lambda: pins.test_elig_matches_episode_sum(True),
    lambda: pins.test_prefix_sum_matches_episode_sum(),
    lambda: pins.test_affine_matches_bruteforce_sum(True, True),
    lambda: pins.test_affine_every_reset_pattern(False),
    lambda: pins.test_affine_grad_matches_finite_differences(False, 0.3),
    lambda: pins.test_affine_grad_matches_finite_differences(True, 0.3),
    lambda: pins.test_affine_tm_matches_bruteforce_on_transpose(True),
    lambda: pins.test_affine_tm_is_row_major_on_transposed_arrays(),
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, tmp_path, monkeypatch):
    before, after = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(before) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(before, after)
    c_path = tmp_path / "mutant.c"
    so_path = tmp_path / "mutant.so"
    c_path.write_text(mutated)
    subprocess.run(["gcc", "-O1", "-fPIC", "-shared", str(c_path), "-o", str(so_path), "-lm"],
                   check=True)
    monkeypatch.setattr(oracle_mod, "_lib", oracle_mod.bind(ctypes.CDLL(str(so_path))))
    caught = 0
    for pin in PIN_TESTS:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin caught mutant {name}"


def test_unmutated_oracle_passes_all_pins():
    for pin in PIN_TESTS:
        pin()
    assert oracle.gae is oracle_mod.gae
