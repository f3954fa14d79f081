"""Plant plausible mistakes in a copy of the oracle's C source, on the CPU, and
check that the pin suite catches every one of them.

Each mutant is oracle.c with one textual edit (a swapped operand, a dropped
term, a wrong sign, an off-by-one in the output index), compiled to a scratch
library; the pin tests of test_oracle_pins.py then run against it and at
least one of them must fail.  This is what makes the pins a check of the
oracle rather than a restatement of it.
"""
import math
import os
import subprocess

import pytest

import oracle
import test_oracle_backward_pins as bpins
import test_oracle_decay_pins as dpins
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.abspath(oracle.__file__)), "oracle.c")

MUTANTS = {
    # minGRU, linear
    "z_and_one_minus_z_swapped": ("double one_minus_z = sigmoid(-k[i]);",
                                  "double one_minus_z = sigmoid(k[i]);"),
    "g_branches_swapped": ("return (x >= 0.0) ? x + 0.5 : sigmoid(x);",
                           "return (x >= 0.0) ? sigmoid(x) : x + 0.5;"),
    "g_offset_sign": ("return (x >= 0.0) ? x + 0.5 : sigmoid(x);",
                      "return (x >= 0.0) ? x - 0.5 : sigmoid(x);"),
    "sigmoid_sign": ("return 1.0 / (1.0 + exp(-x));", "return 1.0 / (1.0 + exp(x));"),
    "h0_dropped": ("prev = h0 ? h0[b * h0_bs + d] : 0.0;", "prev = 0.0;"),
    "state_from_wrong_row": ("prev = h[i - D];", "prev = h[i - 1 < 0 ? 0 : i - 1];"),
    "output_shifted_by_one": ("h[i] = one_minus_z * prev + z * g_act(hx[i]);",
                              "h[i] = prev; (void)(one_minus_z * prev + z * g_act(hx[i]));"),
    # minGRU, log space
    "log_astar_sign": ("a_star[d] += -softplus(k[i]);", "a_star[d] += softplus(k[i]);"),
    "log_z_sign": ("double log_z = -softplus(-k[i]);", "double log_z = -softplus(k[i]);"),
    "log_h0_term_dropped": ("m[d] = log(h0[b * h0_bs + d]);\n                acc[d] = 1.0;",
                            "m[d] = -INFINITY;\n                acc[d] = 0.0;"),
    "log_candidate_branch": ("(x >= 0.0) ? log(x + 0.5) : -softplus(-x);",
                             "(x >= 0.0) ? log(x + 0.5) : -softplus(x);"),
    "log_lse_update": ("acc[d] = acc[d] * exp(m[d] - v) + 1.0;", "acc[d] = acc[d] + 1.0;"),
    # MinMax
    "minmax_min_max_swapped": ("x[i] = fmax(fmin(r[i], state), s[i]);",
                               "x[i] = fmin(fmax(r[i], state), s[i]);"),
    "minmax_r_s_swapped": ("x[i] = fmax(fmin(r[i], state), s[i]);",
                           "x[i] = fmax(fmin(s[i], state), r[i]);"),
    "minmax_x0_dropped": ("state = x0 ? x0[b * x0_bs + d] : 0.0;", "state = 0.0;"),
    # minGRU gradient
    "bwd_dk_sign": ("dk[i] = delta * z * one_minus_z * (g - hprev);",
                    "dk[i] = delta * z * one_minus_z * (hprev - g);"),
    "bwd_dk_missing_gate": ("dk[i] = delta * z * one_minus_z * (g - hprev);",
                            "dk[i] = delta * z * (g - hprev);"),
    "bwd_hprev_off_by_one": ("double hprev = (t > 0) ? h[t - 1] : init;",
                             "double hprev = h[t];"),
    "bwd_gprime_branch": ("double gprime = (x >= 0.0) ? 1.0 : sigmoid(x) * sigmoid(-x);",
                          "double gprime = (x >= 0.0) ? 1.0 : sigmoid(x);"),
    "bwd_state_gradient_gate": ("lam = delta * one_minus_z;", "lam = delta * z;"),
    "bwd_direct_gradient_dropped": ("double delta = gy[i] + lam;\n                double hprev",
                                    "double delta = lam + (t == T - 1 ? gy[i] : 0.0);\n                double hprev"),
    "bwd_forward_without_h0": ("            double prev = init;", "            double prev = 0.0;"),
    # MinMax gradient
    "bwd_minmax_tie_to_r": ("double dm_dr = (r[i] < xprev) ? 1.0 : ((r[i] == xprev) ? 0.5 : 0.0);",
                            "double dm_dr = (r[i] <= xprev) ? 1.0 : 0.0;"),
    "bwd_minmax_tie_to_s": ("double dout_dm = (m > s[i]) ? 1.0 : ((m == s[i]) ? 0.5 : 0.0);",
                            "double dout_dm = (m > s[i]) ? 1.0 : 0.0;"),
    "bwd_minmax_state_path": ("lam = delta * dout_dm * dm_dx;", "lam = delta * dm_dx;"),
    # time decay
    "decay_exponent_sign": ("return (x > 1e4) ? 0.0 : exp(-x);", "return (x > 1e4) ? 0.0 : exp(x);"),
    "decay_gates_the_write": ("h[i] = sigmoid(-k[i]) * (gamma * prev) + sigmoid(k[i]) * g_act(hx[i]);",
                              "h[i] = sigmoid(-k[i]) * prev + gamma * sigmoid(k[i]) * g_act(hx[i]);"),
    "decay_clamp_keeps_state": ("return (x > 1e4) ? 0.0 : exp(-x);", "return (x > 1e4) ? 1.0 : exp(-x);"),
    "decay_log1p_ignored": ("    double u = log1p_delta ? log1p(gap) : gap;\n    double x = lam * u;\n    return (x > 1e4)",
                            "    double u = gap; (void)log1p_delta;\n    double x = lam * u;\n    return (x > 1e4)"),
    "decay_bwd_dk_without_gamma": ("dk[i] = delta * z * one_minus_z * (g - gamma * hprev);",
                                   "dk[i] = delta * z * one_minus_z * (g - hprev);"),
    "decay_bwd_dlam_sign": ("return (x > 1e4) ? 0.0 : -u * exp(-x);", "return (x > 1e4) ? 0.0 : u * exp(-x);"),
    "decay_bwd_state_without_gamma": ("back = delta * one_minus_z * gamma;", "back = delta * one_minus_z;"),
    "bwd_minmax_r_s_swapped": ("dr[i] = delta * dout_dm * dm_dr;\n                ds[i] = delta * dout_ds;",
                               "ds[i] = delta * dout_dm * dm_dr;\n                dr[i] = delta * dout_ds;"),
}


def _pin_checks():
    """Every pin of test_oracle_pins.py, with its parameters spelled out."""
    out = []
    for name in ("mingru_worked_example.txt", "mingru_worked_example_noh0.txt"):
        out.append(lambda n=name: pins.test_mingru_linear_golden(n))
        out.append(lambda n=name: pins.test_mingru_log_golden(n))
    out.append(pins.test_minmax_golden)
    for wh in (False, True):
        for km in (0.0, 2.0, -2.0):
            out.append(lambda a=wh, b=km: pins.test_linear_and_log_space_agree(a, b))
    out += [pins.test_gate_one_gives_candidate, pins.test_large_gate_is_near_candidate,
            pins.test_gate_zero_holds_state, pins.test_small_gate_is_near_state,
            pins.test_sigmoid_branches_match_library, pins.test_positive_and_inside_hull,
            pins.test_minmax_selection_bound_monotone_hold, pins.test_minmax_default_state_is_zero]
    for args in [(math.log(3.0), 0.5, 0.2), (0.3, -1.7, 0.9), (-1.1, 2.25, 0.5)]:
        out.append(lambda a=args: pins.test_constant_inputs_closed_form(*a))
    for T in (1, 2):
        out.append(lambda t=T: pins.test_minmax_brute_force(t))
    # gradient pins
    for shape in [(1, 1, 1), (2, 7, 3)]:
        for wh in (False, True):
            out.append(lambda a=shape, b=wh: bpins.test_mingru_backward_matches_autograd(a, b, 0.0))
    out += [bpins.test_mingru_backward_one_step_closed_form,
            bpins.test_mingru_backward_state_gradient_is_product_of_gates,
            bpins.test_mingru_backward_convex_combination_conserves_gradient,
            bpins.test_mingru_backward_saturated_gates,
            bpins.test_minmax_backward_default_state_is_zero,
            bpins.test_minmax_backward_gradient_weights_are_bounded]
    for seed in range(2):
        out.append(lambda sd=seed: bpins.test_minmax_backward_matches_autograd_with_ties(sd))
        out.append(lambda sd=seed: bpins.test_minmax_backward_conserves_gradient(sd))
    # time-decay pins
    for wh in (False, True):
        out.append(lambda a=wh: dpins.test_zero_gap_and_zero_rate_are_the_plain_recurrence(a))
    out += [dpins.test_wiping_gap_restarts_the_sequence, dpins.test_log1p_delta_compresses_the_gaps,
            dpins.test_decay_backward_lambda_finite_differences,
            dpins.test_decay_backward_without_decay_is_the_plain_gradient]
    for args in [(0.3, 0.7, 0.5, 0.4, 0.8), (-1.2, -0.9, 2.0, 0.1, 0.2)]:
        out.append(lambda a=args: dpins.test_constant_inputs_closed_form(*a))
    for flag in (False, True):
        out.append(lambda f=flag: dpins.test_decay_backward_matches_autograd(f))
    return out


def test_unmutated_oracle_passes_every_check():
    for check in _pin_checks():
        check()


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistake_is_caught(mutant, tmp_path):
    before, after = MUTANTS[mutant]
    src = open(SRC).read()
    assert src.count(before) >= 1, f"mutation anchor for {mutant} not found"
    msrc = tmp_path / "mutant.c"
    msrc.write_text(src.replace(before, after, 1))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", *oracle.CFLAGS, "-o", str(lib), str(msrc), "-lm"], check=True)
    failures = 0
    with oracle.use_library(str(lib)):
        for check in _pin_checks():
            try:
                check()
            except (AssertionError, ValueError, FloatingPointError):
                failures += 1
    assert failures > 0, f"no pin caught mutant {mutant}"
