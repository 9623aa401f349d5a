"""The oracle's pins catch plausible mistakes.

Each case compiles a copy of the oracle's C source with one deliberate
mistake planted (on the CPU, in a temporary directory), loads it in place of
the real oracle and checks that at least one pin test fails.
"""
import os
import subprocess

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "nh_oracle.c")

MUTANTS = {
    "tie_break_to_higher_id": ("return ia < ib;", "return ia > ib;"),
    "group_score_sum": ("if (sel[q * g + i] > m) m = sel[q * g + i];", "m += sel[q * g + i];"),
    "sigmoid_sign": ("s[e] = 1.0 / (1.0 + exp(-l));", "s[e] = 1.0 / (1.0 + exp(l));"),
    "relu_not_squared": ("u[i] = r * r;", "u[i] = r;"),
    "relu_dropped": ("double r = a > 0.0 ? a : 0.0;", "double r = a;"),
    "shared_dropped": ("if (c->n_shared) mlp_relu2", "if (0) mlp_relu2"),
    "e2m1_mantissa_weight": ("1.0 + 0.5 * m, (int)e - 1", "1.0 + 0.25 * m, (int)e - 1"),
    "e2m1_subnormal_wrong": ("(e == 0) ? 0.5 * m :", "(e == 0) ? 1.0 * m :"),
    "e4m3_bias_off_by_one": ("ldexp(1.0 + m / 8.0, (int)e - 7)", "ldexp(1.0 + m / 8.0, (int)e - 8)"),
    "nvfp4_nibble_order": ("(col & 1) ? (byte >> 4) : (byte & 15u)", "(col & 1) ? (byte & 15u) : (byte >> 4)"),
    "nvfp4_scale_group_of_8": ("* w->scale_pitch + col / 16]", "* w->scale_pitch + col / 8]"),
    "nvfp4_global_ignored": ("* (double)w->global[mat];", ";"),
    "norm_ignored": ("w[j] = c->norm ? c->alpha * s[cand[j]] / sum : c->alpha * s[cand[j]];",
                     "w[j] = c->alpha * s[cand[j]];"),
    "alpha_dropped": ("w[j] = c->norm ? c->alpha * s[cand[j]] / sum : c->alpha * s[cand[j]];",
                      "w[j] = c->norm ? s[cand[j]] / sum : s[cand[j]];"),
    "down_transposed": ("wt_get(down, mat, h * down->cols + i)",
                        "wt_get(down, mat, i * down->rows + h)"),
    "weights_from_biased_score": ("for (int64_t j = 0; j < c->k; ++j) sum += s[cand[j]];",
                                  "for (int64_t j = 0; j < c->k; ++j) sum += sel[cand[j]];"),
    "norm_over_k_minus_1": ("for (int64_t j = 0; j < c->k; ++j) sum += s[cand[j]];",
                            "for (int64_t j = 0; j + 1 < c->k; ++j) sum += s[cand[j]];"),
    "bf16_widen_wrong_shift": ("<< 16;", "<< 15;"),
    "top2_sum_takes_group_min": ("gs[q] = sel[tmp[0]] + sel[tmp[1]];",
                                 "gs[q] = sel[tmp[0]] + sel[tmp[g - 1]];"),
    "bias_ignored_in_selection": ("sel[e] = s[e] + (bias ? (double)bias[e] : 0.0);",
                                  "sel[e] = s[e];"),
    "bias_subtracted": ("sel[e] = s[e] + (bias ? (double)bias[e] : 0.0);",
                        "sel[e] = s[e] - (bias ? (double)bias[e] : 0.0);"),
}

PINS = ["tests/test_oracle_route.py", "tests/test_oracle_forward.py",
        "tests/test_oracle_nvfp4.py"]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site of {name} not found"
    mut = tmp_path / "mut.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", str(so),
                           str(mut), "-lm"])
    prev = oracle._swap_library(str(so))
    try:
        rc = pytest.main(["-q", "-x", "-p", "no:cacheprovider", "--no-header", "-o",
                          "addopts=", *[os.path.join(os.path.dirname(HERE), p) for p in PINS]])
    finally:
        oracle._restore_library(prev)
    assert rc != 0, f"no pin failed for mutant {name}"
