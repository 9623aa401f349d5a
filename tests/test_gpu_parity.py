"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle.

Small workloads are compared on every token and span several MMA tiles with
ragged tails; the full-size workloads are compared on their routing (every
token) and on the block output of 256 sampled tokens, every excused and
every exact-tie token, and tokens drawn from every tile of the expert GEMMs'
tile table (both CTAs of a pair tile, first and last rows of a swapped
remainder tile), in the launch configuration the benchmark uses.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import (assert_same_up_to_sum_order, check_output, check_routing, make_block,
                      run_block, sample_tokens, tile_tokens, to_dev)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def small(name, **kw):
    base = dict(name=name, T=300, hidden_size=512, n_routed_experts=16, n_group=4, topk_group=2,
                num_experts_per_tok=4, moe_intermediate_size=320,
                moe_shared_expert_intermediate_size=640, seed=7, wr_std=0.05, w_std=0.05)
    base.update(kw)
    return synth.MoEConfig(**base)


SMALL = {
    # prefill orientation: 128-row tiles, N tails (320 = 256 + 64, 512 = 2 x 256)
    "small_prefill": small("small_prefill"),
    # ragged T, one group, no shared expert, norm off
    "small_noshared": small("small_noshared", T=131, n_group=1, topk_group=1,
                            n_shared_experts=0, norm_topk_prob=False, seed=8),
    # decode orientation with 16 / 32 / 64-row activation tiles
    "small_swap16": small("small_swap16", T=5, seed=9),
    "small_swap32": small("small_swap32", T=29, seed=10),
    "small_swap64": small("small_swap64", T=64, seed=11, moe_intermediate_size=192),
    # float32 CUDA-core path, odd sizes
    "small_f32_odd": small("small_f32_odd", T=77, hidden_size=100, moe_intermediate_size=36,
                           moe_shared_expert_intermediate_size=52, dtype="f32", seed=12),
    # limits: 512 experts, 64 groups, top-32
    "small_max_experts": small("small_max_experts", T=70, hidden_size=128, n_routed_experts=512,
                               n_group=64, topk_group=8, num_experts_per_tok=32,
                               moe_intermediate_size=64, moe_shared_expert_intermediate_size=64,
                               seed=13),
    # NVFP4 weights (W4A16): decode orientation 16 / 32 / 64, and 64-row tiles
    # with a gathered x_perm for T > 64
    "small_nvfp4_t5": small("small_nvfp4_t5", T=5, seed=41, weight_format="nvfp4"),
    "small_nvfp4_t29": small("small_nvfp4_t29", T=29, seed=42, weight_format="nvfp4"),
    "small_nvfp4_t64": small("small_nvfp4_t64", T=64, seed=43, weight_format="nvfp4",
                             moe_intermediate_size=192),
    "small_nvfp4_t150": small("small_nvfp4_t150", T=150, seed=44, weight_format="nvfp4"),
    # selection paths: 128 candidate experts (the ranking pass at its limit)
    # and 256 (the sequential top-k rounds)
    "small_cand128": small("small_cand128", T=45, hidden_size=128, n_routed_experts=256,
                           n_group=2, topk_group=1, num_experts_per_tok=8,
                           moe_intermediate_size=64, moe_shared_expert_intermediate_size=64,
                           seed=15),
    "small_cand256": small("small_cand256", T=20, hidden_size=128, n_routed_experts=512,
                           n_group=2, topk_group=1, num_experts_per_tok=8,
                           moe_intermediate_size=64, moe_shared_expert_intermediate_size=64,
                           seed=16),
    # single expert (routing is trivial)
    "small_one_expert": small("small_one_expert", T=40, n_routed_experts=1, n_group=1,
                              topk_group=1, num_experts_per_tok=1, seed=14),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_block_every_token(name):
    inp = synth.make_inputs(SMALL[name])
    y, idx, w, _ = run_block(inp)
    exc, _, _ = check_routing(inp.cfg, inp.x, inp.w_router, idx, w)
    check_output(inp, y, idx, w, np.arange(inp.cfg.T), exc)


@pytest.mark.parametrize("T", [700, 290, 64 * 5 + 20])
def test_all_tokens_one_expert_set(T):
    """Degenerate routing: a dominant feature sends every token to the same k
    experts (one expert then spans several row tiles).  700 rows per expert
    end in a partial tile of 188 rows (its own swapped tile); 290 rows end in
    34 rows and 340 in 84, attached to the full tile or not (64 is the
    limit)."""
    cfg = small("skew_all", T=T, seed=15)
    inp = synth.make_inputs(cfg)
    inp.x[:, 0] = synth.f32_to_bf16_bits(np.array([4.0], np.float32))[0]
    inp.w_router[:, 1:] *= np.float32(0.1)       # other features: logits within +-0.6
    inp.w_router[:, 0] = 0.0
    # logits 6, 5, 4, 3: well apart, far from sigmoid saturation
    inp.w_router[[1, 2, 3, 0], 0] = [1.5, 1.25, 1.0, 0.75]
    y, idx, w, _ = run_block(inp)
    assert np.all(idx == np.array([1, 2, 3, 0]))
    exc, _, _ = check_routing(cfg, inp.x, inp.w_router, idx, w)
    check_output(inp, y, idx, w, np.arange(cfg.T), exc)


@pytest.mark.parametrize("variant", ["bias", "top2", "bias_top2"])
def test_router_variants(variant):
    """Selection-only correction bias and the top-2-sum group score."""
    cfg = small("variants", T=257, n_routed_experts=64, n_group=8, topk_group=3,
                num_experts_per_tok=6, seed=16, wr_std=0.1)
    gs = 1 if "top2" in variant else 0
    inp = synth.make_inputs(cfg, with_bias="bias" in variant)
    blk = make_block(inp)
    blk.c.group_score = gs
    y, idx, w, _ = run_block(inp, blk)
    exc, _, _ = check_routing(cfg, inp.x, inp.w_router, idx, w, bias=inp.bias, group_score=gs)
    # the block output under the GPU routing (weights from the unbiased scores)
    tok = np.arange(cfg.T)
    ref, _, _ = oracle.forward_parallel(inp, tokens=tok, override_idx=idx,
                                        override_w=w.astype(np.float64))
    assert np.abs(y - ref).max() <= 2e-2 * np.abs(ref).max()


def test_zero_tokens():
    cfg = SMALL["small_prefill"]
    inp = synth.make_inputs(cfg.replace(T=1))
    blk = make_block(inp)
    x = to_dev(inp.x)[:0]
    y = blk.forward(x)
    torch.cuda.synchronize()
    assert y.shape == (0, cfg.H)


def test_host_api_graph_matches_eager():
    """The public call with a host tensor (pinned copies, CUDA graph) equals the
    eager path, up to the order of the combine's float32 adds."""
    inp = synth.make_inputs(SMALL["small_swap16"])
    blk = make_block(inp)
    y_host = blk(inp.x).float().numpy()
    y_eager = blk.forward(to_dev(inp.x)).float().cpu().numpy()
    assert_same_up_to_sum_order(y_host, y_eager, "bf16")
    y2 = blk(inp.x).float().numpy()          # second replay
    assert_same_up_to_sum_order(y2, y_eager, "bf16")
    # another input through the same graph (the staging buffer is refilled)
    x2 = np.ascontiguousarray(inp.x[::-1])
    y3 = blk(x2).float().numpy()
    assert_same_up_to_sum_order(y3, blk.forward(to_dev(x2)).float().cpu().numpy(), "bf16")


@pytest.mark.parametrize("name", ["small_swap16", "small_prefill"])
def test_host_pipeline_matches_eager(name):
    """The pipelined host call (two buffer sets, copies on their own streams)
    gives every batch the result of the eager call, in order."""
    inp = synth.make_inputs(SMALL[name])
    blk = make_block(inp)
    rng = np.random.default_rng(3)
    batches = [inp.x] + [np.ascontiguousarray(inp.x[rng.permutation(inp.x.shape[0])])
                         for _ in range(4)]
    ref = [blk.forward(to_dev(b)).float().cpu().numpy() for b in batches]
    host = [torch.from_numpy(b).view(torch.bfloat16).pin_memory() for b in batches]
    seen = []
    for i, y in blk.pipeline(host):
        seen.append(i)
        assert_same_up_to_sum_order(y.float().numpy(), ref[i], "bf16")
    assert seen == list(range(len(batches)))


@pytest.mark.parametrize("name", ["small_swap16", "small_swap32"])
def test_fused_decode_forward_matches_two_launches(name):
    """For decode batches nh_moe_forward runs the up and down projections as one
    persistent launch (the down tiles of a tile entry wait for its up tiles).
    Called twice after one permute, it gives the y_acc of the separate
    experts_up + experts_down launches, up to float32 summation order."""
    import non_gated_relu_b200 as nh
    inp = synth.make_inputs(SMALL[name])
    blk = make_block(inp)
    x = to_dev(inp.x)
    T = x.shape[0]
    b = blk.buffers(T)
    blk.forward(x, b)
    fused = [torch.zeros_like(b.y_acc) for _ in range(2)]
    for acc in fused:
        nh.forward(blk.c, x, blk.w_up, blk.w_down, b.ws, acc)
    two = torch.zeros_like(b.y_acc)
    nh.experts_up(blk.c, x, blk.w_up, b.ws)
    nh.experts_down(blk.c, T, blk.w_down, b.ws, two)
    torch.cuda.synchronize()
    assert blk.check(T) == 0
    ref = two.cpu().numpy()
    assert np.abs(ref).max() > 0
    for acc in fused:
        assert_same_up_to_sum_order(acc.cpu().numpy(), ref, "f32")
    L = nh.workspace_layout(blk.c, T)
    ready = b.ws.view(torch.uint8)[L.ready:L.ready + 4 * L.max_tiles]
    assert (ready == 0).all(), "a fused launch leaves its ready counters zero"


@pytest.mark.parametrize("name", ["small_nvfp4_t5", "small_nvfp4_t29"])
def test_fused_nvfp4_decode_forward_repeats(name):
    """For NVFP4 decode batches nh_moe_forward_nvfp4 runs both projections as one
    launch of the rows GEMV (down tasks wait for their entry's up tasks).  Called
    twice after one permute it gives the same y_acc up to float32 summation
    order, matches the block (whose output the oracle checks), and leaves its
    ready counters zero."""
    import non_gated_relu_b200 as nh
    inp = synth.make_inputs(SMALL[name])
    blk = make_block(inp)
    x = to_dev(inp.x)
    T = x.shape[0]
    b = blk.buffers(T)
    blk.forward(x, b)
    torch.cuda.synchronize()
    ref = b.y_acc.cpu().numpy().copy()
    outs = []
    for _ in range(2):
        acc = torch.zeros_like(b.y_acc)
        if blk.has_shared:
            nh.shared_nvfp4(blk.c, x, blk.q4["shared_up"], blk.q4["shared_down"], acc, b.ws_shared)
        nh.forward_nvfp4(blk.c, x, blk.q4["up"], blk.q4["down"], b.ws, acc)
        outs.append(acc)
    torch.cuda.synchronize()
    assert blk.check(T) == 0
    for acc in outs:
        assert_same_up_to_sum_order(acc.cpu().numpy(), ref, "f32")
    L = nh.workspace_layout(blk.c, T)
    ready = b.ws.view(torch.uint8)[L.ready:L.ready + 4 * L.max_tiles]
    assert (ready == 0).all(), "a fused launch leaves its ready counters zero"


@pytest.mark.parametrize("name", ["small_prefill", "small_swap16", "small_f32_odd"])
def test_shared_store_equals_add_into_zeros(name):
    """nh_moe_shared_store writes the shared expert as y_acc's starting value:
    bit-equal to nh_moe_shared adding into zeros (each element is computed once,
    and 0 + v == v), whatever y_acc held before."""
    import non_gated_relu_b200 as nh
    inp = synth.make_inputs(SMALL[name])
    blk = make_block(inp)
    x = to_dev(inp.x)
    T = x.shape[0]
    b = blk.buffers(T)
    added = torch.zeros_like(b.y_acc)
    nh.shared(blk.c, x, blk.w_shared_up, blk.w_shared_down, added, b.ws_shared)
    stored = torch.full_like(b.y_acc, float("nan"))
    nh.shared_store(blk.c, x, blk.w_shared_up, blk.w_shared_down, stored, b.ws_shared)
    torch.cuda.synchronize()
    assert torch.equal(stored, added)
    assert added.abs().max().item() > 0


# ----------------------------------------------------------------------------- full size
FULL = synth.CONFIG_ORDER


def full_inputs(name):
    cfg = synth.CONFIGS[name]
    b = None
    if cfg.skew_hot_groups:
        import json, os
        with open(os.path.join(os.path.dirname(__file__), "golden",
                               "skew_prefill_t2048.json")) as f:
            b = json.load(f)["b"]
    return synth.make_inputs(cfg, skew_b=b)


@pytest.mark.parametrize("name", FULL)
def test_full_workload(name):
    inp = full_inputs(name)
    cfg = inp.cfg
    y, idx, w, blk = run_block(inp)
    exc, _, _ = check_routing(cfg, inp.x, inp.w_router, idx, w, tie_tokens=inp.tie_tokens)
    if cfg.T <= 64:
        tokens = np.arange(cfg.T)
    else:
        # 256 sampled tokens, every excused and every exact-tie token, and
        # tokens that cover every tile of the expert GEMMs' tile table
        extra = list(np.nonzero(exc)[0])
        if inp.tie_tokens is not None:
            extra += list(inp.tie_tokens)
        covered, n_tiles, n_swapped = (tile_tokens(blk, cfg.T) if not blk.latent
                                       else (np.zeros(0, np.int64), 0, 0))
        if cfg.dtype == "bf16" and not blk.latent and cfg.weight_format == "native":
            assert n_tiles >= -(-cfg.T * cfg.k // 256) and len(covered) > 0
        tokens = sample_tokens(cfg.T, 256, seed=cfg.seed, extra=extra + list(covered))
        print(f"{name}: {len(tokens)} tokens compared ({n_tiles} tiles, {n_swapped} "
              f"swapped remainder tiles covered), {int(exc.sum())} excused")
    check_output(inp, y, idx, w, tokens, exc)
    if inp.tie_tokens is not None:
        # exact ties: lowest-index picks, equal weights alpha / k
        np.testing.assert_allclose(w[inp.tie_tokens], cfg.routed_scaling_factor / cfg.k,
                                   rtol=1e-6)
    # the CUDA-graph replay of the same call gives the same result, up to the
    # order of the combine's float32 atomic adds
    graph, xs, yg = blk.capture(cfg.T)
    xs.copy_(to_dev(inp.x))
    graph.replay()
    torch.cuda.synchronize()
    assert_same_up_to_sum_order(yg.float().cpu().numpy(), y, cfg.dtype)
