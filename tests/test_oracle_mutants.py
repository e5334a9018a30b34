"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
in a temporary directory), loads the mutant in place of the oracle and runs
the pin tests that should notice it.  A pin set that lets a mutant through is
too weak.  The real oracle is restored after each case.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "lapsum_oracle.c")

# (name, original text, planted mistake, pin tests that must fail on it)
MUTANTS = [
    ("cdf_upper_sign", "1.0 - 0.5 * exp(-x)", "1.0 - 0.5 * exp(x)",
     [lambda: pins.test_budget_and_probabilities("normal", 10, 0.1)]),
    ("sign_dropped_half", "c - 0.5 * exp(U) + 0.5 * exp(L)", "c - exp(U) + 0.5 * exp(L)",
     [lambda: pins.test_bisection_matches_segment_brute_force(1)]),
    ("sign_flip_tie_branch", "if (L > U) return 1;", "if (L < U) return 1;",
     [pins.test_sign_function_on_flat_plateau]),
    ("bisection_direction", "if (sg > 0) lo = mid;", "if (sg < 0) lo = mid;",
     [lambda: pins.test_bisection_matches_segment_brute_force(1)]),
    ("upper_bound_log", "log((double)n / (2.0 * k))", "log((double)n / (4.0 * k))",
     [pins.test_single_score_closed_form]),
    ("vjp_missing_inv_t", "g[i] = (f / t) * (v[i] - R);", "g[i] = f * (v[i] - R);",
     [lambda: pins.test_vjp_central_finite_differences(0, 12, 3.0, 0.5)]),
    ("vjp_t_sign", "*g_t = -(1.0 / t) * 0.5", "*g_t = (1.0 / t) * 0.5",
     [lambda: pins.test_vjp_kt_central_finite_differences(0, 12, 3.0, 0.5)]),
    ("vjp_t_drops_mean", "(a3 - a1 * a2 / a0)", "(a3)",
     [lambda: pins.test_vjp_kt_central_finite_differences(0, 12, 3.0, 0.5)]),
    ("vjp_unweighted_mean", "swv += w * v[i];", "swv += v[i];",
     [lambda: pins.test_vjp_identities(0)]),
    ("vjp_abs_dropped", "double f = 0.5 * exp(-fabs(r[i] - b) / t);",
     "double f = 0.5 * exp(-(r[i] - b) / t);",
     [lambda: pins.test_vjp_central_finite_differences(1, 40, 7.5, 0.2)]),
    ("noise_scale", "t * log(1.0 - 2.0 * fabs(u))", "t * log(1.0 - fabs(u))",
     [pins.test_sample_noise_is_laplace_and_indices_uniform]),
    ("rank_off_by_one", "if (sf <= alpha) h = c;", "if (sf <= alpha) h = c + 1;",
     [lambda: pins.test_binomial_ranks_match_scipy(1000, 0.5, 0.05)]),
    ("fold_tail_sign", "sr += exp(-(r[i] - aR) / t);", "sr += exp((r[i] - aR) / t);",
     [pins.test_fold_reconstructs_budget_inside_bracket]),
    ("splitmix_constant", "0xBF58476D1CE4E5B9ull", "0xBF58476D1CE4E5B8ull",
     [pins.test_splitmix64_published_vector]),
    ("hard_rank_floor", "(int64_t)ceil(k);", "(int64_t)floor(k) + 1;",
     [pins.test_hard_topk_worked_cases]),
    ("hard_tie_share", "frac = (k - (double)a) / (double)m;",
     "frac = (k - (double)a) / (double)(m + 1);",
     [pins.test_hard_topk_worked_cases]),
    ("hard_midpoint", "b = 0.5 * (c + d);", "b = c;",
     [lambda: pins.test_hard_topk_is_the_soft_solution_at_tiny_temperature(0, 40, 7.0, 0.0)]),
    ("order_stat_index", "*aR = (l >= 1) ? s[m - l] : INFINITY;",
     "*aR = (l >= 1) ? s[m - l - 1] : INFINITY;",
     [pins.test_bracket_order_statistics]),
]


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


@pytest.mark.parametrize("name,orig,bad,checks", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, source, name, orig, bad, checks):
    assert source.count(orig) == 1, f"mutation site for {name} not unique"
    mutated = source.replace(orig, bad)
    c_path = tmp_path / "mutant.c"
    so_path = tmp_path / "mutant.so"
    c_path.write_text(mutated)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-o",
                    str(so_path), str(c_path), "-lm"], check=True)
    real = oracle._lib()
    oracle._LIB = oracle.configure(ctypes.CDLL(str(so_path)))
    try:
        caught = 0
        for check in checks:
            try:
                check()
            except (AssertionError, oracle.OracleError):
                caught += 1
        assert caught == len(checks), f"mutant {name} passed a pin meant to catch it"
    finally:
        oracle._LIB = real
