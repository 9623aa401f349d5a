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
    "norm_ignored": ("w[j] = c->norm ? c->alpha * s[cand[j]] / sum : c->alpha * s[cand[j]];",
                     "w[j] = c->alpha * s[cand[j]];"),
    "alpha_dropped": ("w[j] = c->norm ? c->alpha * s[cand[j]] / sum : c->alpha * s[cand[j]];",
                      "w[j] = c->norm ? s[cand[j]] / sum : s[cand[j]];"),
    "down_transposed": ("load(wd, wd_off + h * wd_stride + i, c->dtype)",
                        "load(wd, wd_off + i * c->H + h, c->dtype)"),
    "weights_from_biased_score": ("for (int64_t j = 0; j < c->k; ++j) sum += s[cand[j]];",
                                  "for (int64_t j = 0; j < c->k; ++j) sum += sel[cand[j]];"),
    "norm_over_k_minus_1": ("for (int64_t j = 0; j < c->k; ++j) sum += s[cand[j]];",
                            "for (int64_t j = 0; j + 1 < c->k; ++j) sum += s[cand[j]];"),
    "bf16_widen_wrong_shift": ("<< 16;", "<< 15;"),
}

PINS = ["tests/test_oracle_route.py", "tests/test_oracle_forward.py"]


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
