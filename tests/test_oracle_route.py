"""Pins of the oracle's routing against values that do not come from the oracle.

* a hand-worked four-token example (tests/golden/route_hand_example.json);
* brute force over every group subset and every expert subset on tiny inputs
  with many exact ties (an enumeration, independent of the oracle's sorts);
* the special case n_group = 1, which is plain top-k (numpy stable argsort);
* invariants on random inputs: weights sum to routed_scaling_factor, chosen
  experts lie in the chosen groups, the chosen groups carry the topk_group
  largest group maxima, the unchosen candidates score no higher than the
  k-th pick.
Logits in the pins are built exactly representable (identity router, small
dyadic values), so the selection can be checked on logits: the sigmoid is
strictly increasing and preserves their order.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from synth import MoEConfig

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny_cfg(E, G, tg, k, H=None, norm=True, alpha=2.5):
    return MoEConfig("t", T=1, hidden_size=H or E, n_routed_experts=E, n_group=G,
                     topk_group=tg, num_experts_per_tok=k, moe_intermediate_size=4,
                     moe_shared_expert_intermediate_size=4, dtype="f32",
                     norm_topk_prob=norm, routed_scaling_factor=alpha)


def test_hand_example():
    with open(os.path.join(GOLDEN, "route_hand_example.json")) as f:
        g = json.load(f)
    c = g["config"]
    cfg = tiny_cfg(c["n_routed_experts"], c["n_group"], c["topk_group"],
                   c["num_experts_per_tok"], alpha=c["routed_scaling_factor"])
    L = math.log(3.0)
    x = np.array([[v * L for v in t["x_in_units_of_L"]] for t in g["tokens"]], np.float32)
    wr = np.eye(8, dtype=np.float32)
    idx, w, gg, ge = oracle.route(cfg, x, wr)
    for n, t in enumerate(g["tokens"]):
        assert idx[n].tolist() == t["topk_idx"], t["name"]
        np.testing.assert_allclose(w[n], t["topk_w"], rtol=0, atol=g["tolerance_w"])
    # token B and D have exact ties at the group stage: the gap is zero, not excused
    assert gg[1] == 0.0 and gg[3] == 0.0


def brute_force(l, E, G, tg, k):
    """Enumerate every tg-subset of groups, then every k-subset of their experts.

    The pick maximises the descending-sorted score vector lexicographically
    (groups by their maxima first, then experts); equal vectors go to the
    lexicographically smallest index tuple.  Output order (score desc, id asc).
    """
    g = E // G
    gmax = [max(l[q * g:(q + 1) * g]) for q in range(G)]

    def better(va, ta, vb, tb):
        return va > vb or (va == vb and ta < tb)

    bestQ = bestv = None
    for Q in itertools.combinations(range(G), tg):
        v = sorted((gmax[q] for q in Q), reverse=True)
        if bestQ is None or better(v, Q, bestv, bestQ):
            bestQ, bestv = Q, v
    cand = [q * g + i for q in bestQ for i in range(g)]
    bestK = bestv = None
    for K in itertools.combinations(sorted(cand), k):
        v = sorted((l[e] for e in K), reverse=True)
        if bestK is None or better(v, K, bestv, bestK):
            bestK, bestv = K, v
    return sorted(bestK, key=lambda e: (-l[e], e))


def _tiny_cases(n, seed):
    rng = np.random.default_rng(seed)
    shapes = [(4, 2), (4, 4), (6, 3), (8, 4), (8, 2), (12, 3), (12, 4), (16, 4), (16, 8), (6, 1)]
    for _ in range(n):
        E, G = shapes[rng.integers(len(shapes))]
        g = E // G
        tg = int(rng.integers(1, G + 1))
        k = int(rng.integers(1, tg * g + 1))
        yield E, G, tg, k


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_with_ties(seed):
    vals = np.array([-2.0, -1.0, -0.5, 0.0, 0.5, 1.0, 2.0], np.float32)
    for E, G, tg, k in _tiny_cases(40, seed):
        cfg = tiny_cfg(E, G, tg, k)
        rng = np.random.default_rng([seed, E, G, tg, k])
        # few distinct values -> many exact ties at both stages
        x = vals[rng.integers(0, 3 + seed % 4, size=(24, E))]
        idx, w, _, _ = oracle.route(cfg, x, np.eye(E, dtype=np.float32))
        for t in range(x.shape[0]):
            want = brute_force(x[t].astype(np.float64), E, G, tg, k)
            assert idx[t].tolist() == want, (E, G, tg, k, x[t])
            np.testing.assert_allclose(w[t].sum(), 2.5, rtol=1e-12)


def test_brute_force_random_router():
    """Continuous logits through a dense router (no ties); H != E."""
    rng = np.random.default_rng(11)
    for E, G, tg, k in _tiny_cases(30, 99):
        H = 24
        cfg = tiny_cfg(E, G, tg, k, H=H)
        x = rng.standard_normal((16, H)).astype(np.float32)
        wr = (rng.standard_normal((E, H)) * 0.3).astype(np.float32)
        idx, _, _, _ = oracle.route(cfg, x, wr)
        l = x.astype(np.float64) @ wr.astype(np.float64).T
        for t in range(16):
            assert idx[t].tolist() == brute_force(l[t], E, G, tg, k)


def test_single_group_is_plain_topk():
    rng = np.random.default_rng(5)
    for E, k in [(16, 2), (32, 6), (64, 8), (7, 7)]:
        cfg = tiny_cfg(E, 1, 1, k, H=40)
        x = rng.standard_normal((50, 40)).astype(np.float32)
        wr = (rng.standard_normal((E, 40)) * 0.2).astype(np.float32)
        # quantise a third of the logits to produce ties: dyadic router rows
        wr[::3] = np.round(wr[::3] * 4) / 4
        x[::2] = np.round(x[::2])
        idx, _, _, _ = oracle.route(cfg, x, wr)
        l = x.astype(np.float64) @ wr.astype(np.float64).T
        s = 1.0 / (1.0 + np.exp(-l))
        want = np.argsort(-s, axis=1, kind="stable")[:, :k]
        np.testing.assert_array_equal(idx, want)


@pytest.mark.parametrize("norm", [True, False])
def test_invariants_random(norm):
    rng = np.random.default_rng(7)
    for E, G, tg, k in [(128, 8, 1, 6), (256, 8, 2, 8), (64, 8, 3, 5), (32, 4, 2, 8)]:
        H = 64
        cfg = tiny_cfg(E, G, tg, k, H=H, norm=norm)
        x = rng.standard_normal((200, H)).astype(np.float32)
        wr = (rng.standard_normal((E, H)) * 0.2).astype(np.float32)
        idx, w, gg, ge = oracle.route(cfg, x, wr)
        l = x.astype(np.float64) @ wr.astype(np.float64).T
        s = 1.0 / (1.0 + np.exp(-l))
        g = E // G
        for t in range(200):
            sel = idx[t]
            assert len(set(sel.tolist())) == k
            gmax = s[t].reshape(G, g).max(axis=1)
            chosen_groups = set((sel // g).tolist())
            assert len(chosen_groups) <= tg
            top_groups = np.argsort(-gmax, kind="stable")[:tg]
            assert chosen_groups <= set(top_groups.tolist())
            kth = s[t, sel].min()
            cand = [q * g + i for q in top_groups for i in range(g)]
            rest = [e for e in cand if e not in set(sel.tolist())]
            if rest:
                assert s[t, rest].max() <= kth
            assert np.all(np.diff(s[t, sel]) <= 0)           # output order
            if norm:
                assert abs(w[t].sum() - 2.5) < 1e-12
                np.testing.assert_allclose(w[t], 2.5 * s[t, sel] / s[t, sel].sum(), rtol=1e-12)
            else:
                np.testing.assert_allclose(w[t], 2.5 * s[t, sel], rtol=1e-12)
            assert gg[t] >= 0 and ge[t] >= 0


def test_gaps_report_near_ties():
    cfg = tiny_cfg(8, 4, 1, 2)
    x = np.zeros((2, 8), np.float32)
    x[0, 0] = 1.0
    x[0, 2] = np.nextafter(np.float32(1.0), np.float32(0))   # group 1 max just below group 0
    x[1, 0] = 1.0
    x[1, 1] = 1.0                                             # exact tie inside the chosen group
    _, _, gg, ge = oracle.route(cfg, x, np.eye(8, dtype=np.float32))
    assert 0 < gg[0] < 1e-7
    assert ge[1] == 0.0


def test_correction_bias_selects_but_does_not_weight():
    """With a bias the selection uses s + b, the weights the unbiased s."""
    cfg = tiny_cfg(8, 4, 1, 2)
    x = np.zeros((1, 8), np.float32)
    x[0, 0] = 1.0                    # s0 = sigmoid(1) ~ 0.731, all others 0.5
    b = np.zeros(8, np.float32)
    b[5] = 0.5                       # group 2 wins with 1.0 > 0.731
    idx, w, _, _ = oracle.route(cfg, x, np.eye(8, dtype=np.float32), bias=b)
    assert idx[0].tolist() == [5, 4]
    np.testing.assert_allclose(w[0], [1.25, 1.25], rtol=1e-12)


def test_group_score_top2_sum_variant():
    cfg = tiny_cfg(8, 2, 1, 2)
    x = np.zeros((1, 8), np.float32)
    x[0, 0] = 3.0                    # group 0: one high expert, rest low
    x[0, 1:4] = -3.0
    x[0, 4:8] = 1.0                  # group 1: four medium experts
    wr = np.eye(8, dtype=np.float32)
    idx_max, _, _, _ = oracle.route(cfg, x, wr, group_score=0)
    idx_sum, _, _, _ = oracle.route(cfg, x, wr, group_score=1)
    assert idx_max[0].tolist() == [0, 1]
    assert idx_sum[0].tolist() == [4, 5]


def test_bad_configs_rejected():
    assert oracle.check_config(tiny_cfg(8, 3, 1, 2)) != 0     # E % G
    assert oracle.check_config(tiny_cfg(8, 4, 5, 2)) != 0     # tg > G
    assert oracle.check_config(tiny_cfg(8, 4, 1, 3)) != 0     # k > tg * g
    assert oracle.check_config(tiny_cfg(8, 4, 1, 2)) == 0


def brute_force_variant(l, b, E, G, tg, k, top2, alpha=2.5):
    """Enumeration for the router variants: selection scores s + b (b the
    correction bias), group score the max or the sum of the two largest
    selection scores of the group; the weights use the unbiased s."""
    s = 1.0 / (1.0 + np.exp(-l))
    sel = s + b
    g = E // G

    def gscore(q):
        v = sorted(sel[q * g:(q + 1) * g], reverse=True)
        return v[0] + v[1] if top2 else v[0]

    def better(va, ta, vb, tb):
        return va > vb or (va == vb and ta < tb)

    bestQ = bestv = None
    for Q in itertools.combinations(range(G), tg):
        v = sorted((gscore(q) for q in Q), reverse=True)
        if bestQ is None or better(v, Q, bestv, bestQ):
            bestQ, bestv = Q, v
    cand = [q * g + i for q in bestQ for i in range(g)]
    bestK = bestv = None
    for K in itertools.combinations(sorted(cand), k):
        v = sorted((sel[e] for e in K), reverse=True)
        if bestK is None or better(v, K, bestv, bestK):
            bestK, bestv = K, v
    picks = sorted(bestK, key=lambda e: (-sel[e], e))
    ssum = sum(s[e] for e in picks)
    return picks, [alpha * s[e] / ssum for e in picks]


@pytest.mark.parametrize("top2", [0, 1])
@pytest.mark.parametrize("seed", range(3))
def test_brute_force_router_variants(seed, top2):
    """Correction bias (selection only) and the top-2-sum group score against
    enumeration, with exact ties in the logits and in the bias."""
    vals = np.array([-2.0, -1.0, -0.5, 0.0, 0.5, 1.0, 2.0], np.float32)
    bvals = np.array([0.0, 0.25, 0.5], np.float32)
    n = 0
    for E, G, tg, k in _tiny_cases(60, 100 + seed):
        if top2 and E // G < 2:
            continue
        cfg = tiny_cfg(E, G, tg, k)
        rng = np.random.default_rng([seed, top2, E, G, tg, k])
        x = vals[rng.integers(0, 3 + seed % 4, size=(16, E))]
        b = bvals[rng.integers(0, 3, size=E)]
        idx, w, _, _ = oracle.route(cfg, x, np.eye(E, dtype=np.float32), bias=b,
                                    group_score=top2)
        for t in range(x.shape[0]):
            want, wt = brute_force_variant(x[t].astype(np.float64), b.astype(np.float64),
                                           E, G, tg, k, top2)
            assert idx[t].tolist() == want, (E, G, tg, k, x[t], b)
            np.testing.assert_allclose(w[t], wt, rtol=1e-12)
        n += 1
    assert n >= 20
