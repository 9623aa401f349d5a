"""Tensor-parallel sharding on the CPU (no GPU).

* the 64-feature block partition of I and S covers every feature once, in
  order, with shares that differ by at most one block;
* the oracle run on each rank's weight slices sums, over the ranks, to the
  oracle run on the whole block (exact up to float64 rounding): the slices
  cut the right rows of fc1 / shared up_proj and the right columns of
  fc2 / shared down_proj, for dense and for NVFP4 weights (whose column cut
  also re-pads the scale rows);
* two gloo ranks each compute their partial with the oracle and sum it with
  the same all-reduce helper the GPU block uses.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth
from non_gated_relu_b200 import tp
from synth import MoEConfig


def small_cfg(**kw):
    base = dict(name="tp", T=10, hidden_size=128, n_routed_experts=8, n_group=4, topk_group=2,
                num_experts_per_tok=3, moe_intermediate_size=192,
                moe_shared_expert_intermediate_size=320, seed=31, wr_std=0.2, w_std=0.05)
    base.update(kw)
    return MoEConfig(**base)


@pytest.mark.parametrize("n,world", [(64, 1), (192, 2), (192, 3), (1856, 2), (1856, 8),
                                     (3712, 8), (640, 4)])
def test_shard_range_partition(n, world):
    ranges = [tp.shard_range(n, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == n
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0                                  # contiguous, in rank order
    sizes = [b - a for a, b in ranges]
    assert all(s > 0 and s % tp.BLOCK == 0 for s in sizes)
    assert max(sizes) - min(sizes) <= tp.BLOCK


def test_shard_range_rejects():
    with pytest.raises(ValueError):
        tp.shard_range(100, 2, 0)                        # not whole blocks
    with pytest.raises(ValueError):
        tp.shard_range(128, 3, 0)                        # fewer blocks than ranks
    with pytest.raises(ValueError):
        tp.shard_range(128, 2, 2)                        # no such rank


def test_nemotron_shapes_shard():
    cfg = synth.CONFIGS["decode_bf16_t8"]
    assert [tp.shard_config(cfg, 2, r).moe_intermediate_size for r in range(2)] == [896, 960]
    assert [tp.shard_config(cfg, 2, r).moe_shared_expert_intermediate_size
            for r in range(2)] == [1856, 1856]


def _rank_inputs(inp, world, rank):
    cfg_r = tp.shard_config(inp.cfg, world, rank)
    kw = dict(cfg=cfg_r, x=inp.x, w_router=inp.w_router, bias=inp.bias)
    if inp.nvfp4 is not None:
        q = tp.shard_nvfp4(inp.cfg, world, rank, inp.nvfp4)
        return synth.MoEInputs(w_up=None, w_down=None, w_shared_up=None, w_shared_down=None,
                               nvfp4=q, **kw)
    up, down, su, sd = tp.shard_weights(inp.cfg, world, rank, inp.w_up, inp.w_down,
                                        inp.w_shared_up, inp.w_shared_down)
    return synth.MoEInputs(w_up=up, w_down=down, w_shared_up=su, w_shared_down=sd, **kw)


@pytest.mark.parametrize("fmt", ["native", "nvfp4"])
@pytest.mark.parametrize("world", [2, 3])
def test_sum_of_rank_partials_is_the_block(world, fmt):
    cfg = small_cfg(dtype="bf16", weight_format=fmt)
    inp = synth.make_inputs(cfg)
    y, idx, w = oracle.forward(inp)
    total = np.zeros_like(y)
    for r in range(world):
        yr, idx_r, w_r = oracle.forward(_rank_inputs(inp, world, r))
        np.testing.assert_array_equal(idx_r, idx)        # the router is replicated
        np.testing.assert_array_equal(w_r, w)
        total += yr
    np.testing.assert_allclose(total, y, rtol=1e-12, atol=1e-13 * np.abs(y).max())


def test_a_wrong_cut_is_caught():
    """The pin above fails when a rank takes the wrong rows of fc1."""
    cfg = small_cfg(dtype="bf16")
    inp = synth.make_inputs(cfg)
    y, _, _ = oracle.forward(inp)
    total = np.zeros_like(y)
    for r in range(2):
        ri = _rank_inputs(inp, 2, r)
        ri.w_up = np.ascontiguousarray(ri.w_up[:, ::-1, :])   # rows of fc1 reversed
        total += oracle.forward(ri)[0]
    assert np.abs(total - y).max() > 1e-3 * np.abs(y).max()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = small_cfg(dtype="bf16")
        inp = synth.make_inputs(cfg)
        yr, _, _ = oracle.forward(_rank_inputs(inp, world, rank))
        t = torch.from_numpy(yr)
        tp.all_reduce_sum(t)
        q.put((rank, t.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_all_reduce_the_partials():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    y, _, _ = oracle.forward(synth.make_inputs(small_cfg(dtype="bf16")))
    for r in range(world):
        np.testing.assert_allclose(out[r], y, rtol=1e-12, atol=1e-13 * np.abs(y).max())
