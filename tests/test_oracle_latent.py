"""Pins of the oracle's latent block (routed experts between fc1_latent_proj
and fc2_latent_proj).

The pages name the two projections and give no formula, so the reading
itself is unpinned; what these tests fix is that the oracle computes that
reading:
* identity projections (L = H) give the plain block, bit for bit;
* a permutation P as fc1, P^T as fc2 and the experts' weights permuted to
  match give the plain block up to the float64 summation order (P is not
  symmetric, so a transposed projection fails);
* with L < H the result equals a dense float64 composition, and routing
  follows the full-width x.
"""
import numpy as np
import pytest

import oracle
import synth
from synth import MoEConfig


def cfg_of(**kw):
    base = dict(name="lat", T=9, hidden_size=64, n_routed_experts=8, n_group=4, topk_group=2,
                num_experts_per_tok=3, moe_intermediate_size=48,
                moe_shared_expert_intermediate_size=32, seed=61, wr_std=0.2, w_std=0.1,
                dtype="f32")
    base.update(kw)
    return MoEConfig(**base)


def plain_and_latent(perm, n_shared=1):
    """The plain block and a latent block (L = H) with fc1 = P, fc2 = P^T and the
    experts' weights permuted so that both compute the same function."""
    cfg = cfg_of(n_shared_experts=n_shared)
    inp = synth.make_inputs(cfg)
    H = cfg.H
    P = np.eye(H, dtype=np.float32)[perm]                 # (P x)[l] = x[perm[l]]
    lcfg = cfg.replace(latent_size=H)
    lat = synth.MoEInputs(
        cfg=lcfg, x=inp.x, w_router=inp.w_router,
        w_up=np.ascontiguousarray(inp.w_up[:, :, perm]),          # W_up P^T
        w_down=np.ascontiguousarray(inp.w_down[:, perm, :]),      # P W_down
        w_shared_up=inp.w_shared_up, w_shared_down=inp.w_shared_down,
        w_latent_fc1=P, w_latent_fc2=np.ascontiguousarray(P.T))
    return inp, lat


@pytest.mark.parametrize("n_shared", [1, 0])
def test_identity_projections_give_the_plain_block(n_shared):
    inp, lat = plain_and_latent(np.arange(64), n_shared)
    y0, i0, w0 = oracle.forward(inp)
    y1, i1, w1 = oracle.forward(lat)
    np.testing.assert_array_equal(i1, i0)
    np.testing.assert_array_equal(w1, w0)
    np.testing.assert_array_equal(y1, y0)


def test_permutation_projections_give_the_plain_block():
    perm = np.random.default_rng(3).permutation(64)
    assert (perm != np.argsort(perm)).any()               # P is not symmetric
    inp, lat = plain_and_latent(perm)
    y0, _, _ = oracle.forward(inp)
    y1, _, _ = oracle.forward(lat)
    # the experts' inner sums run in permuted order: equal to float64 rounding
    np.testing.assert_allclose(y1, y0, rtol=1e-12, atol=1e-13 * np.abs(y0).max())
    # fc1 and fc2 swapped (a transposed reading) gives something else
    bad = synth.MoEInputs(**{**lat.__dict__, "w_latent_fc1": lat.w_latent_fc2,
                             "w_latent_fc2": lat.w_latent_fc1})
    y2, _, _ = oracle.forward(bad)
    assert np.abs(y2 - y0).max() > 1e-3 * np.abs(y0).max()


def relu2(a):
    return np.maximum(a, 0.0) ** 2


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_reduced_width_matches_dense_composition(dtype):
    cfg = cfg_of(dtype=dtype, latent_size=32)
    inp = synth.make_inputs(cfg)
    assert inp.w_up.shape == (8, 48, 32) and inp.w_latent_fc1.shape == (32, 64)
    y, idx, w = oracle.forward(inp)
    f = lambda a: synth.to_f64(a, dtype)
    x = f(inp.x)
    # routing is the plain block's (on the full-width x)
    plain = synth.MoEInputs(cfg.replace(latent_size=0), inp.x, inp.w_router,
                            np.zeros((8, 48, 64), inp.w_up.dtype),
                            np.zeros((8, 64, 48), inp.w_up.dtype), inp.w_shared_up,
                            inp.w_shared_down)
    _, idx0, w0 = oracle.forward(plain)
    np.testing.assert_array_equal(idx, idx0)
    np.testing.assert_array_equal(w, w0)
    xl = x @ f(inp.w_latent_fc1).T
    want = relu2(x @ f(inp.w_shared_up).T) @ f(inp.w_shared_down).T
    for t in range(cfg.T):
        yl = np.zeros(32)
        for j in range(cfg.k):
            e = idx[t, j]
            yl += w[t, j] * (relu2(f(inp.w_up[e]) @ xl[t]) @ f(inp.w_down[e]).T)
        want[t] += f(inp.w_latent_fc2) @ yl
    np.testing.assert_allclose(y, want, rtol=1e-10, atol=1e-12 * np.abs(want).max())
