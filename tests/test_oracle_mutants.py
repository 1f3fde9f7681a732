"""The oracle's pins are sensitive: plant one plausible mistake at a time in a copy of the
oracle (on the CPU), rebuild it, and check that at least one pin in test_oracle_pins fails.

Each mutation is a mistake someone writing the Sparse GQA definition could make: a reversed
tie rule, the own block not counted in the budget, a lost causal limit, the wrong softmax
scale, a flipped gate sign, an off-by-one in the candidate range, a dropped term in the block
mean, an interleaved head->group mapping, or the wrong group's index query; and in the Gated
SWA definition, a window one key too long or too short, unscaled scores, a missing gate or an
interleaved head->group mapping (these are checked against the SWA pins); and in the token
coverage of the ablation, a reversed ranking, an interleaved head->group mapping, ties sent to
the higher token, a top set one token short, and the query's own token left out (these are
checked against the coverage pins); and in the FP8 KV storage, ties rounded away from even, a
scale one power of two off either way, the subnormal range cut at the wrong binade, and a dropped
sign (checked against the FP8 pins); and in the backward, the softmax Jacobian's subtracted term
dropped, dk unscaled, dv ungated, the gate's derivative without (1 - s) (backward pins).
"""
import os
import subprocess

import pytest

import oracle
import tests.test_oracle_pins as pins

MUTANTS = {
    "tie_to_higher_block": ("return a.s > b.s || (a.s == b.s && a.j < b.j);",
                            "return a.s > b.s || (a.s == b.s && a.j > b.j);"),
    "own_block_not_in_budget": ("const int m = std::min(Kb - 1, c);", "const int m = std::min(Kb, c);"),
    "no_causal_limit": ("u < (j + 1) * dm->B && u <= t;", "u < (j + 1) * dm->B;"),
    "scale_by_index_dim": ("1.0 / std::sqrt((double)d);", "1.0 / std::sqrt((double)dm->d_idx);"),
    "gate_sign": ("std::exp(-gl)", "std::exp(gl)"),
    "complete_own_block_is_candidate": ("const int c = t / dm->B;                  //",
                                        "const int c = (t + 1) / dm->B;            //"),
    "dropped_term_in_mean": ("for (int r = 0; r < dm->B; ++r)", "for (int r = 0; r < dm->B - 1 + (dm->B == 1); ++r)"),
    "interleaved_heads": ("const int h = (int)(rh % dm->Hq), g = h / R;\n    const long b = rows_bt[2 * row];\n    const int t = rows_bt[2 * row + 1];\n    const int32_t* S",
                          "const int h = (int)(rh % dm->Hq), g = h % dm->G;\n    const long b = rows_bt[2 * row];\n    const int t = rows_bt[2 * row + 1];\n    const int32_t* S"),
    "wrong_group_query": ("q_idx + rg * dm->d_idx", "q_idx + row * dm->G * dm->d_idx"),
}

PIN_CALLS = [
    lambda: pins.test_brute_force_small(None, 8, 40),
    lambda: pins.test_brute_force_small(None, 1, 13),
    lambda: pins.test_brute_force_batch2_uneven(None),
    lambda: pins.test_dense_reduction_matches_sdpa(None, 96, 8, 8, 2, 16),
    lambda: pins.test_hand_worked_example(None),
    lambda: pins.test_compress_closed_forms(None),
    lambda: pins.test_first_token_is_gated_v0(None),
    lambda: pins.test_selection_invariants(None, 8, 24),
    lambda: pins.test_exact_ties_go_to_lower_block(None),
]


# Gated SWA: a window one key too long or too short, no softmax scale, no gate, the wrong group
SWA_MUTANTS = {
    "swa_window_one_longer": ("const int u_lo = std::max(0, t - window + 1);",
                              "const int u_lo = std::max(0, t - window);"),
    "swa_window_one_shorter": ("const int u_lo = std::max(0, t - window + 1);",
                               "const int u_lo = std::max(0, t - window + 2);"),
    "swa_unscaled_scores": ("z[u - u_lo] = dot * inv_sqrt_d;", "z[u - u_lo] = dot;"),
    "swa_no_gate": ("out[rh * d + e] = (o[e] / l) * (1.0 / (1.0 + std::exp(-gl)));", "out[rh * d + e] = (o[e] / l);"),
    "swa_interleaved_heads": ("const int h = (int)(rh % dm->Hq), g = h / R;\n    const long b = rows_bt[2 * row];\n    const int t = rows_bt[2 * row + 1];\n    const int u_lo",
                              "const int h = (int)(rh % dm->Hq), g = h % dm->G;\n    const long b = rows_bt[2 * row];\n    const int t = rows_bt[2 * row + 1];\n    const int u_lo"),
}


# Token coverage: each mutation touches only oracle_coverage (its anchors occur nowhere else)
COVERAGE_MUTANTS = {
    "coverage_ascending_rank": (
        "if (n < t + 1) std::nth_element(z.begin(), z.begin() + n, z.end(), ranks_before);",
        "if (n < t + 1) std::nth_element(z.begin(), z.begin() + n, z.end(),\n"
        "        [](const Cand& a, const Cand& b) { return a.s < b.s || (a.s == b.s && a.j < b.j); });"),
    "coverage_interleaved_heads": (
        "const int h = (int)(rh % dm->Hq), g = h / R;\n    const long b = rows_bt[2 * row];\n"
        "    const int t = rows_bt[2 * row + 1];\n    std::vector<char> in_sel",
        "const int h = (int)(rh % dm->Hq), g = h % dm->G;\n    const long b = rows_bt[2 * row];\n"
        "    const int t = rows_bt[2 * row + 1];\n    std::vector<char> in_sel"),
    "coverage_ties_to_higher_token": (
        "if (n < t + 1) std::nth_element(z.begin(), z.begin() + n, z.end(), ranks_before);",
        "if (n < t + 1) std::nth_element(z.begin(), z.begin() + n, z.end(),\n"
        "        [](const Cand& a, const Cand& b) { return a.s > b.s || (a.s == b.s && a.j > b.j); });"),
    "coverage_top_set_one_short": ("const int n = std::min(ktop, t + 1);", "const int n = std::min(ktop, t);"),
    "coverage_own_token_left_out": ("std::vector<Cand> z(t + 1);\n    for (int u = 0; u <= t; ++u) {",
                                    "std::vector<Cand> z(t + 1);\n    for (int u = 0; u < t; ++u) {"),
}


# FP8 KV storage: rounding ties away from even, a scale one power too small or too large, the
# subnormal range cut at the wrong binade, a dropped sign
FP8_MUTANTS = {
    "fp8_ties_away_from_even": ("if (frac > 0.5 || (frac == 0.5 && std::fmod(r, 2.0) != 0.0)) r += 1.0;",
                                "if (frac >= 0.5) r += 1.0;"),
    "fp8_scale_one_too_small": ("while (amax <= 448.0 * std::ldexp(1.0, e - 1)) --e;",
                                "while (amax <= 448.0 * std::ldexp(1.0, e - 1)) --e;\n      --e;"),
    "fp8_scale_one_too_large": ("while (amax <= 448.0 * std::ldexp(1.0, e - 1)) --e;",
                                "while (amax <= 448.0 * std::ldexp(1.0, e - 1)) --e;\n      ++e;"),
    "fp8_subnormal_binade": ("if (E < -6) E = -6;", "if (E < -7) E = -7;"),
    "fp8_sign_dropped": ("return (c & 0x80) ? -mag : mag;", "return mag;"),
}


def _fp8_pin_calls():
    import tests.test_oracle_fp8_pins as fp8
    return [
        lambda: fp8.test_fp8_codes_match_torch_e4m3_cast(None),
        lambda: fp8.test_fp8_scale_is_the_smallest_power_of_two(None),
        lambda: fp8.test_fp8_closed_forms(None),
        lambda: fp8.test_fp8_error_bound_and_bf16_exactness(None),
    ]


# Backward: the softmax Jacobian's subtracted term dropped, dk without the 1/sqrt(d) scale, dv from
# dy instead of dy * sigmoid(gate), the gate's derivative without its (1 - s) factor
BACKWARD_MUTANTS = {
    "bw_no_softmax_correction": ("const double dz = p[n] * (dp[n] - sum_pdp);", "const double dz = p[n] * dp[n];"),
    "bw_dk_unscaled": ("dk[kvrow + e] += dz * bf16_to_f64(qv[e]) * inv_sqrt_d;",
                       "dk[kvrow + e] += dz * bf16_to_f64(qv[e]);"),
    "bw_dv_ungated": ("dov[e] = dye * s;", "dov[e] = dye;"),
    "bw_gate_derivative": ("dgate[rh * d + e] = dye * o[e] * s * (1.0 - s);", "dgate[rh * d + e] = dye * o[e] * s;"),
}


def _backward_pin_calls():
    import tests.test_oracle_backward_pins as bw
    return [
        lambda: bw.test_backward_dense_reduction_matches_sdpa_autograd(None, 40, 8),
        lambda: bw.test_backward_sparse_selection_matches_masked_autograd(None),
        lambda: bw.test_backward_matches_finite_differences_of_the_forward(None),
    ]


def _coverage_pin_calls():
    return [
        lambda: pins.test_coverage_brute_force(None, False),
        lambda: pins.test_coverage_brute_force(None, True),
        lambda: pins.test_coverage_all_scores_tied_takes_lowest_tokens(None),
        lambda: pins.test_coverage_closed_forms(None),
    ]


def _swa_pin_calls():
    import tests.test_oracle_swa_pins as swa
    return [
        lambda: swa.test_swa_brute_force(None, 40, 8, 13),
        lambda: swa.test_swa_brute_force(None, 33, 1, 5),
        lambda: swa.test_swa_full_window_is_dense_causal(None, 70, 8, 2, 16),
        lambda: swa.test_swa_block_aligned_window_equals_block_selection(None),
        lambda: swa.test_swa_locality(None),
    ]


ALL_MUTANTS = {**MUTANTS, **SWA_MUTANTS, **COVERAGE_MUTANTS, **FP8_MUTANTS, **BACKWARD_MUTANTS}


@pytest.mark.parametrize("name", sorted(ALL_MUTANTS))
def test_pins_catch_mutant(tmp_path, name):
    old, new = ALL_MUTANTS[name]
    calls = (PIN_CALLS if name in MUTANTS else _swa_pin_calls() if name in SWA_MUTANTS
             else _coverage_pin_calls() if name in COVERAGE_MUTANTS
             else _fp8_pin_calls() if name in FP8_MUTANTS else _backward_pin_calls())
    src = open(oracle.SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {name}"
    if name in COVERAGE_MUTANTS or name in FP8_MUTANTS or name in BACKWARD_MUTANTS:
        assert src.count(old) == 1, f"mutation anchor not unique: {name}"
    mutated = src.replace(old, new)
    cpp = tmp_path / "mut.cpp"
    so = tmp_path / "libmut.so"
    cpp.write_text(mutated)
    subprocess.run(["g++", "-O2", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC", "-o", str(so), str(cpp)],
                   check=True)
    saved = oracle._lib
    oracle._lib = oracle.load(str(so))
    caught = []
    try:
        for call in calls:
            try:
                call()
            except (AssertionError, ValueError) as e:
                caught.append(type(e).__name__)
    finally:
        oracle._lib = saved
    assert caught, f"no pin caught mutant {name}"
