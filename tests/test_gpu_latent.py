"""Latent blocks on the GPU, through the C ABI, against the oracle.

The routed experts run in width L between fc1_latent_proj and
fc2_latent_proj (nh_moe_latent_in / nh_moe_latent_out around the unchanged
routed path in its expert-width config); routing and the shared expert see
the full-width x.  The GPU rounds x_lat and the combined y_lat to the
activation dtype (they are Linear inputs; the oracle rounds nothing), which
the bf16 tolerance covers.
"""
import numpy as np
import pytest

import synth
from gpu_util import check_output, check_routing, run_block

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def small(name, **kw):
    base = dict(name=name, T=150, hidden_size=256, n_routed_experts=16, n_group=4, topk_group=2,
                num_experts_per_tok=4, moe_intermediate_size=192,
                moe_shared_expert_intermediate_size=320, seed=71, wr_std=0.05, w_std=0.05,
                latent_size=128)
    base.update(kw)
    return synth.MoEConfig(**base)


CASES = {
    "latent_prefill": small("latent_prefill"),
    "latent_decode": small("latent_decode", T=6, seed=72),
    "latent_t40": small("latent_t40", T=40, seed=73, latent_size=192),
    "latent_noshared": small("latent_noshared", T=70, seed=74, n_shared_experts=0),
    "latent_nvfp4": small("latent_nvfp4", T=6, seed=75, weight_format="nvfp4"),
    "latent_f32": small("latent_f32", T=33, seed=76, dtype="f32", latent_size=96),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_latent_block_matches_oracle(name):
    cfg = CASES[name]
    inp = synth.make_inputs(cfg)
    y, idx, w, blk = run_block(inp)
    exc, _, _ = check_routing(cfg, inp.x, inp.w_router, idx, w)
    check_output(inp, y, idx, w, np.arange(cfg.T), exc)
    # the latent projections change the result (not a pass-through)
    assert blk.latent and np.abs(y).max() > 0


def test_routed_calls_reject_the_full_latent_config():
    import non_gated_relu_b200 as nh
    cfg = CASES["latent_decode"]
    inp = synth.make_inputs(cfg)
    blk = nh.NemotronHMoE(cfg, inp.w_router, inp.w_up, inp.w_down, inp.w_shared_up,
                          inp.w_shared_down, w_latent_fc1=inp.w_latent_fc1,
                          w_latent_fc2=inp.w_latent_fc2)
    b = blk.buffers(cfg.T)
    with pytest.raises(nh.NHMoEError) as e:
        nh.permute(blk.c, b.x_lat, b.topk_idx, b.topk_w, b.ws)
    assert e.value.status == nh.NH_ERR_INVALID_ARG
