"""Pins of the oracle's NVFP4 weight decode (W4A16, group size 16).

* every E2M1 code and a set of E4M3 scale codes against values written out by
  hand from the formats' bit fields (tests/golden/nvfp4_codes.json);
* the layout: even column in the low nibble, one scale byte per 16 columns,
  padded scale rows, one global scale per matrix;
* the input encoder's round trip stays within the format's resolution;
* the block output with NVFP4 weights equals a dense numpy float64 forward on
  the decoded weights (pins which matrix / row / column each weight feeds).
"""
import json
import os

import numpy as np
import pytest

import oracle
import synth
from synth import MoEConfig

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden():
    with open(os.path.join(GOLDEN, "nvfp4_codes.json")) as f:
        return json.load(f)


def pack(codes):
    """codes uint8 [..., cols] (4-bit) -> packed [..., cols/2], even column low."""
    codes = np.asarray(codes, np.uint8)
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def test_e2m1_codes():
    g = golden()["e2m1"]
    codes = np.arange(16, dtype=np.uint8)[None, None, :]        # one row of 16 columns
    scales = np.zeros((1, 1, 16), np.uint8)
    scales[..., 0] = 56                                          # E4M3 1.0
    deq = oracle.dequant_nvfp4((pack(codes), scales, np.ones(1, np.float32)), 1, 16)
    np.testing.assert_array_equal(deq[0], [g[str(c)] for c in range(16)])


def test_e4m3_scales():
    g = golden()["e4m3"]
    names = sorted(g, key=int)
    rows = len(names)
    codes = np.full((1, rows, 16), 2, np.uint8)                  # E2M1 1.0 everywhere
    scales = np.zeros((1, rows, 16), np.uint8)
    for r, c in enumerate(names):
        scales[0, r, 0] = int(c)
    deq = oracle.dequant_nvfp4((pack(codes), scales, np.ones(1, np.float32)), rows, 16)
    for r, c in enumerate(names):
        np.testing.assert_array_equal(deq[r], np.full(16, g[c]))
    scales[0, 0, 0] = 0x7F                                       # S.1111.111 is NaN
    deq = oracle.dequant_nvfp4((pack(codes), scales, np.ones(1, np.float32)), rows, 16)
    assert np.isnan(deq[0]).all()


def test_layout_nibbles_groups_padding_global():
    rows, cols = 3, 48
    rng = np.random.default_rng(1)
    codes = rng.integers(0, 16, size=(2, rows, cols)).astype(np.uint8)
    pitch = synth.nvfp4_scale_pitch(cols)
    assert pitch == 16
    scales = np.full((2, rows, pitch), 0xFF, np.uint8)           # padding bytes are NaN codes
    sc = rng.choice([48, 56, 60, 64], size=(2, rows, cols // 16)).astype(np.uint8)
    scales[..., : cols // 16] = sc
    glob = np.array([0.5, 3.0], np.float32)
    e2m1 = golden()["e2m1"]
    e4m3 = golden()["e4m3"]
    for mat in (0, 1):
        deq = oracle.dequant_nvfp4((pack(codes), scales, glob), rows, cols, mat=mat)
        want = np.array([[e2m1[str(codes[mat, r, c])] * e4m3[str(sc[mat, r, c // 16])] * glob[mat]
                          for c in range(cols)] for r in range(rows)])
        np.testing.assert_array_equal(deq, want)


def test_encoder_round_trip():
    rng = np.random.default_rng(2)
    w = (rng.standard_normal((2, 16, 64)) * 0.02).astype(np.float32)
    q = synth.quantize_nvfp4(w)
    for mat in (0, 1):
        deq = oracle.dequant_nvfp4(q, 16, 64, mat=mat)
        blocks_w = w[mat].reshape(16, 4, 16).astype(np.float64)
        blocks_d = deq.reshape(16, 4, 16)
        scale = np.abs(blocks_d).max(axis=-1, keepdims=True) / 6.0  # exact block scale x global
        # each decoded element is the nearest E2M1 grid point (within rounding of
        # the E4M3 scale, so allow one half spacing of the coarsest step, 2 units)
        err = np.abs(blocks_w - blocks_d)
        assert np.all(err <= 1.0 * scale + 1e-12)
        rel = np.sqrt(np.mean((blocks_w - blocks_d) ** 2) / np.mean(blocks_w ** 2))
        assert rel < 0.12


def small_q4_cfg(**kw):
    base = dict(name="q4", T=12, hidden_size=64, n_routed_experts=8, n_group=4, topk_group=2,
                num_experts_per_tok=3, moe_intermediate_size=32,
                moe_shared_expert_intermediate_size=48, seed=23, wr_std=0.2, w_std=0.1,
                weight_format="nvfp4")
    base.update(kw)
    return MoEConfig(**base)


def mlp(x, wu, wd):
    return (np.maximum(x @ wu.T, 0.0) ** 2) @ wd.T


@pytest.mark.parametrize("n_shared", [1, 0])
def test_forward_matches_dense_decoded(n_shared):
    cfg = small_q4_cfg(n_shared_experts=n_shared)
    inp = synth.make_inputs(cfg)
    y, idx, w = oracle.forward(inp)
    x = synth.to_f64(inp.x, cfg.dtype)
    q = inp.nvfp4
    want = np.zeros_like(y)
    if n_shared:
        want += mlp(x, oracle.dequant_nvfp4(q["shared_up"], cfg.S, cfg.H),
                    oracle.dequant_nvfp4(q["shared_down"], cfg.H, cfg.S))
    for e in range(cfg.E):
        f = mlp(x, oracle.dequant_nvfp4(q["up"], cfg.I, cfg.H, mat=e),
                oracle.dequant_nvfp4(q["down"], cfg.H, cfg.I, mat=e))
        wt = np.where(idx == e, w, 0.0).sum(axis=1)
        want += wt[:, None] * f
    np.testing.assert_allclose(y, want, rtol=1e-11, atol=1e-12 * np.abs(want).max())
