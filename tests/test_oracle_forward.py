"""Pins of the oracle's block output and permute.

* n_routed_experts = 1, top-1, norm on: the block is alpha * a dense relu^2 MLP
  plus the shared expert -> numpy float64 matmuls;
* top-k = all experts, one group, norm off: every expert weighted by
  alpha * sigmoid(logit);
* a dense masked formulation y = sum_e W[t, e] f_e(x_t) + shared, with W the
  dense [T, E] routing matrix: pins the gather and the weighted combine;
* equivariance: permuting tokens permutes y; doubling alpha doubles the
  routed part; a routing override reproduces the oracle's own routing;
* bf16 storage is widened exactly;
* the permute against a hand-worked example and invariants.
"""
import json
import os

import numpy as np
import pytest

import oracle
import synth
from synth import MoEConfig

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small_cfg(**kw):
    base = dict(name="s", T=40, hidden_size=48, n_routed_experts=8, n_group=4, topk_group=2,
                num_experts_per_tok=3, moe_intermediate_size=20,
                moe_shared_expert_intermediate_size=28, dtype="f32", seed=21,
                wr_std=0.2, w_std=0.1)
    base.update(kw)
    return MoEConfig(**base)


def f64(a, cfg):
    return synth.to_f64(a, cfg.dtype)


def mlp(x, wu, wd):
    u = x @ wu.T
    return (np.maximum(u, 0.0) ** 2) @ wd.T


def shared(inp):
    c = inp.cfg
    if not c.n_shared_experts:
        return 0.0
    return mlp(f64(inp.x, c), f64(inp.w_shared_up, c), f64(inp.w_shared_down, c))


def test_single_expert_is_dense_mlp():
    cfg = small_cfg(n_routed_experts=1, n_group=1, topk_group=1, num_experts_per_tok=1)
    inp = synth.make_inputs(cfg)
    y, idx, w = oracle.forward(inp)
    x = f64(inp.x, cfg)
    want = 2.5 * mlp(x, f64(inp.w_up[0], cfg), f64(inp.w_down[0], cfg)) + shared(inp)
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    assert np.all(idx == 0) and np.allclose(w, 2.5)


def test_all_experts_no_norm():
    cfg = small_cfg(n_group=1, topk_group=1, num_experts_per_tok=8, norm_topk_prob=False)
    inp = synth.make_inputs(cfg)
    y, _, _ = oracle.forward(inp)
    x = f64(inp.x, cfg)
    l = x @ inp.w_router.astype(np.float64).T
    s = 1.0 / (1.0 + np.exp(-l))
    want = shared(inp) + sum(2.5 * s[:, e:e + 1] * mlp(x, f64(inp.w_up[e], cfg),
                                                       f64(inp.w_down[e], cfg))
                             for e in range(8))
    np.testing.assert_allclose(y, want, rtol=1e-11, atol=1e-12 * np.abs(want).max())


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("n_shared", [1, 0])
def test_dense_masked_combine(dtype, n_shared):
    cfg = small_cfg(dtype=dtype, n_shared_experts=n_shared)
    inp = synth.make_inputs(cfg)
    y, idx, w = oracle.forward(inp)
    x = f64(inp.x, cfg)
    dense = np.zeros((cfg.T, cfg.E))
    for t in range(cfg.T):
        dense[t, idx[t]] = w[t]
    want = shared(inp) + sum(dense[:, e:e + 1] * mlp(x, f64(inp.w_up[e], cfg),
                                                     f64(inp.w_down[e], cfg))
                             for e in range(cfg.E))
    np.testing.assert_allclose(y, want, rtol=1e-11, atol=1e-12 * np.abs(want).max())


def test_token_permutation_equivariance():
    cfg = small_cfg()
    inp = synth.make_inputs(cfg)
    y, _, _ = oracle.forward(inp)
    p = np.random.default_rng(3).permutation(cfg.T)
    inp2 = synth.MoEInputs(cfg, np.ascontiguousarray(inp.x[p]), inp.w_router, inp.w_up,
                           inp.w_down, inp.w_shared_up, inp.w_shared_down)
    y2, _, _ = oracle.forward(inp2)
    np.testing.assert_array_equal(y2, y[p])
    # a token subset gives the same rows
    sub = np.array([5, 0, 39, 17])
    y3, _, _ = oracle.forward(inp, tokens=sub)
    np.testing.assert_array_equal(y3, y[sub])


def test_alpha_scales_routed_part():
    cfg = small_cfg()
    inp = synth.make_inputs(cfg)
    y1, _, _ = oracle.forward(inp)
    inp2 = synth.MoEInputs(cfg.replace(routed_scaling_factor=5.0), inp.x, inp.w_router,
                           inp.w_up, inp.w_down, inp.w_shared_up, inp.w_shared_down)
    y2, _, _ = oracle.forward(inp2)
    sh = shared(inp)
    np.testing.assert_allclose(y2 - sh, 2.0 * (y1 - sh), rtol=1e-10,
                               atol=1e-12 * np.abs(y1).max())


def test_override_routing():
    cfg = small_cfg()
    inp = synth.make_inputs(cfg)
    y, idx, w = oracle.forward(inp)
    y2, idx2, w2 = oracle.forward(inp, override_idx=idx, override_w=w)
    np.testing.assert_array_equal(y, y2)
    # a different routing gives the dense-masked result of that routing
    idx3 = (idx + 1) % cfg.E
    y3, _, _ = oracle.forward(inp, override_idx=idx3, override_w=w)
    x = f64(inp.x, cfg)
    want = shared(inp).copy()
    for t in range(cfg.T):
        for j in range(cfg.k):
            e = idx3[t, j]
            want[t] += w[t, j] * mlp(x[t:t + 1], f64(inp.w_up[e], cfg), f64(inp.w_down[e], cfg))[0]
    np.testing.assert_allclose(y3, want, rtol=1e-11, atol=1e-12 * np.abs(want).max())


def test_parallel_matches_serial():
    cfg = small_cfg(T=37)
    inp = synth.make_inputs(cfg)
    y, i, w = oracle.forward(inp)
    y2, i2, w2 = oracle.forward_parallel(inp, threads=4)
    np.testing.assert_array_equal(y, y2)
    np.testing.assert_array_equal(i, i2)
    r = oracle.route(cfg, inp.x, inp.w_router)
    r2 = oracle.route_parallel(cfg, inp.x, inp.w_router, threads=3)
    for a, b in zip(r, r2):
        np.testing.assert_array_equal(a, b)


def test_permute_hand_example():
    with open(os.path.join(GOLDEN, "permute_hand_example.json")) as f:
        g = json.load(f)
    p = oracle.permute(np.array(g["topk_idx"]), np.array(g["topk_w"]), g["E"])
    for key in ("counts", "offsets", "perm_token", "perm_slot", "inv_row"):
        np.testing.assert_array_equal(p[key], np.array(g[key]), err_msg=key)
    np.testing.assert_array_equal(p["perm_w"], np.array(g["perm_w"]))


def test_permute_invariants():
    rng = np.random.default_rng(0)
    T, k, E = 300, 6, 32
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    w = rng.random((T, k))
    p = oracle.permute(idx, w, E)
    rows = np.arange(T * k)
    seg = np.searchsorted(p["offsets"], rows, side="right") - 1
    assert np.all(idx[p["perm_token"], p["perm_slot"]] == seg)           # right segment
    assert np.all(p["inv_row"][p["perm_token"], p["perm_slot"]] == rows)  # inverse
    assert np.all(np.diff(p["perm_token"])[np.diff(seg) == 0] > 0)        # stable (t increasing)
    np.testing.assert_array_equal(p["counts"], np.bincount(idx.reshape(-1), minlength=E))
    # the whole order is numpy's stable sort of the (token, slot) assignments by expert
    np.testing.assert_array_equal(p["perm_token"] * k + p["perm_slot"],
                                  np.argsort(idx.reshape(-1), kind="stable"))
