"""Tensor-parallel shards on one GPU, through the C ABI, against the oracle.

Each rank of a world of 2 or 3 runs the whole path on its 64-feature blocks
of I and S (its float32 accumulator y_acc is its contribution).  The
ranks do not wait on one another, so they run one after the other on the
same GPU; the test adds their float32 partials (what the all-reduce does)
and nh_moe_finalize rounds the sum once.  The result must match the
oracle like the unsharded block, and the unsharded GPU block closely.
"""
import numpy as np
import pytest

import synth
from gpu_util import check_output, check_routing, run_block, sample_tokens, to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def small(name, **kw):
    base = dict(name=name, T=150, hidden_size=256, n_routed_experts=16, n_group=4, topk_group=2,
                num_experts_per_tok=4, moe_intermediate_size=448,
                moe_shared_expert_intermediate_size=320, seed=51, wr_std=0.05, w_std=0.05)
    base.update(kw)
    return synth.MoEConfig(**base)


CASES = {
    "tp_prefill": (small("tp_prefill"), (2, 3)),
    "tp_decode": (small("tp_decode", T=6, seed=52), (2, 3)),
    "tp_nvfp4": (small("tp_nvfp4", T=6, seed=53, weight_format="nvfp4"), (2, 3)),
    "tp_noshared": (small("tp_noshared", T=40, n_shared_experts=0, seed=54), (2,)),
    "tp_f32": (small("tp_f32", T=33, dtype="f32", seed=55), (2,)),
}


def tp_run(inp, world):
    from non_gated_relu_b200 import tp
    x = to_dev(inp.x)
    ranks = [tp.TPNemotronHMoE(inp.cfg, inp.w_router, inp.w_up, inp.w_down, inp.w_shared_up,
                               inp.w_shared_down, bias=inp.bias, nvfp4=inp.nvfp4,
                               world=world, rank=r) for r in range(world)]
    parts = [rk.partial(x).clone() for rk in ranks]
    total = parts[0]
    for p in parts[1:]:
        total += p
    y = ranks[0].output(total)
    torch.cuda.synchronize()
    for rk in ranks:
        assert rk.block.check(x.shape[0]) == 0
    b = ranks[0].block.buffers(x.shape[0])
    return (y.float().cpu().numpy().astype(np.float64), b.topk_idx.cpu().numpy(),
            b.topk_w.cpu().numpy())


@pytest.mark.parametrize("name", sorted(CASES))
def test_tp_shards_match_oracle(name):
    cfg, worlds = CASES[name]
    inp = synth.make_inputs(cfg)
    y_full, _, _, _ = run_block(inp)
    for world in worlds:
        y, idx, w = tp_run(inp, world)
        exc, _, _ = check_routing(cfg, inp.x, inp.w_router, idx, w)
        check_output(inp, y, idx, w, np.arange(cfg.T), exc)
        # and close to the unsharded block (only the summation order differs)
        tol = 1e-2 if cfg.dtype == "bf16" else 1e-5
        assert np.abs(y - y_full).max() <= tol * np.abs(y_full).max()


def test_tp_decode_full_size():
    """Nemotron-H decode shapes, 2 ranks: I = 1856 splits 896 / 960."""
    cfg = synth.CONFIGS["decode_bf16_t8"]
    inp = synth.make_inputs(cfg)
    y, idx, w = tp_run(inp, 2)
    exc, _, _ = check_routing(cfg, inp.x, inp.w_router, idx, w)
    check_output(inp, y, idx, w, sample_tokens(cfg.T, 8, 1), exc)
