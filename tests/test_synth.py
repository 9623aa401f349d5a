"""Seeded input generator: determinism, bf16 rounding, tie and skew structure."""
import json
import os

import numpy as np

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_bf16_rounding_nearest_even():
    # bf16 keeps 7 fraction bits: one ulp at 1.0 is 2^-7
    f = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 3 * 2 ** -9, -2.5, 0.0,
                  1.0 + 2 ** -9], np.float32)
    b = synth.f32_to_bf16_bits(f)
    back = synth.bf16_bits_to_f32(b)
    # half-ulp ties go to the even neighbour (1.0 and 1+2^-6); 0.75 ulp rounds up
    np.testing.assert_array_equal(back, np.array([1.0, 1.0, 1.0 + 2 ** -6, 1.0 + 2 ** -7, -2.5,
                                                  0.0, 1.0], np.float32))


def test_deterministic_and_independent_streams():
    cfg = synth.CONFIGS["tiny_f32_t64"]
    a = synth.make_inputs(cfg)
    b = synth.make_inputs(cfg, threads=1)
    for n in ("x", "w_router", "w_up", "w_down", "w_shared_up", "w_shared_down"):
        np.testing.assert_array_equal(getattr(a, n), getattr(b, n))
    up3, down3 = synth.make_expert(cfg, 3)
    np.testing.assert_array_equal(up3, a.w_up[3])
    np.testing.assert_array_equal(down3, a.w_down[3])
    assert a.x.dtype == np.float32 and a.x.shape == (64, 256)
    assert abs(float(a.w_up.std()) - 0.02) < 0.002


def test_bf16_workload_shapes():
    cfg = synth.CONFIGS["decode_bf16_t8"].replace(n_routed_experts=8, n_group=4)
    x, wr, _, _, _ = synth.make_router_and_x(cfg)
    assert x.dtype == np.uint16 and x.shape == (8, 2688)
    assert wr.dtype == np.float32 and wr.shape == (8, 2688)


def test_tie_tokens_tie_exactly():
    cfg = synth.CONFIGS["stress_bf16_t4096"].replace(T=400)
    x, wr, _, ties, tcols = synth.make_router_and_x(cfg)
    assert len(ties) == 20
    xf = synth.to_f64(x, "bf16")
    for t in ties:
        nz = np.nonzero(xf[t])[0]
        assert len(nz) == 1 and nz[0] in tcols
        l = xf[t] @ wr.astype(np.float64).T
        # products of a bf16 value and +-2^-4 / +-2^-5 are exact: the top logit is shared
        assert np.sum(l == l.max()) >= 8
    idx, _, gg, ge = oracle.route(cfg, x, wr)
    assert np.all(ge[ties] == 0.0)


def test_skew_calibration_record():
    with open(os.path.join(GOLDEN, "skew_prefill_t2048.json")) as f:
        rec = json.load(f)
    cfg = synth.CONFIGS["prefill_skewed_bf16_t2048"]
    x, wr, hot, _, _ = synth.make_router_and_x(cfg, skew_b=rec["b"])
    assert hot.tolist() == rec["hot_experts"]
    xf = synth.to_f64(x, "bf16")
    assert np.all(xf[:, -1] == 1.0)
    assert np.all(wr[hot, -1] == np.float32(rec["b"]))
    assert 0.29 <= rec["hot_share"] <= 0.31
