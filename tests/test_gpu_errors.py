"""Failure detection on the GPU, without faulting it.

* a bounded device wait that nothing satisfies runs out, records
  NH_ERR_TIMEOUT in the status word and returns; the context stays usable;
* an expert id out of range reaching the permute is caught by the kernel's
  own bounds check (NH_ERR_DEVICE_CHECK) and skipped;
* a fused decode launch whose down tiles wait on up tiles that can never
  complete them (the ready counters set out of reach) runs out of its bounded
  wait, records NH_ERR_TIMEOUT and returns;
* argument errors are reported before anything is enqueued.
"""
import numpy as np
import pytest

import synth
from gpu_util import make_block, run_block, to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import non_gated_relu_b200 as nh  # noqa: E402


def small_cfg(T=40):
    return synth.MoEConfig("err", T=T, hidden_size=128, n_routed_experts=8, n_group=4,
                           topk_group=2, num_experts_per_tok=2, moe_intermediate_size=64,
                           moe_shared_expert_intermediate_size=128, seed=3, wr_std=0.1)


def test_bounded_wait_times_out_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    nh.selftest_timeout(ws, 20_000_000)          # 20 ms
    assert nh.check_device(ws) == nh.NH_ERR_TIMEOUT
    assert "wait ran out" in nh.last_error()
    # the context is still usable: a full block call works and is clean
    inp = synth.make_inputs(small_cfg())
    y, idx, w, _ = run_block(inp)
    assert np.isfinite(y).all()


def test_out_of_range_expert_id_is_caught_on_device():
    cfg = small_cfg()
    inp = synth.make_inputs(cfg)
    blk = make_block(inp)
    T = cfg.T
    b = blk.buffers(T)
    x = to_dev(inp.x)
    nh.route(blk.c, x, blk.w_router, None, b.topk_idx, b.topk_w, b.ws)
    b.topk_idx[3, 1] = cfg.E + 5                 # corrupt one routing id
    nh.permute(blk.c, x, b.topk_idx, b.topk_w, b.ws)
    assert nh.check_device(b.ws) == nh.NH_ERR_DEVICE_CHECK
    # the next block call starts clean (route clears the status word)
    y, _, _, _ = run_block(inp, blk)
    assert np.isfinite(y).all()


@pytest.mark.parametrize("fmt", ["bf16", "nvfp4"])
def test_fused_decode_wait_times_out(fmt):
    """A decode batch runs the up and down projections as one launch whose down
    tasks wait (bounded) for their tile entry's up tasks.  With the entry
    counters set far below zero after the permute, the waits can never end:
    the launch must record NH_ERR_TIMEOUT and return, and the next block call
    must run clean (the launch leaves its counters zero)."""
    cfg = small_cfg(T=8)
    if fmt == "nvfp4":
        import dataclasses
        cfg = dataclasses.replace(cfg, weight_format="nvfp4")
    inp = synth.make_inputs(cfg)
    blk = make_block(inp)
    T = cfg.T
    b = blk.buffers(T)
    x = to_dev(inp.x)
    nh.route_permute(blk.c, x, blk.w_router, None, b.topk_idx, b.topk_w, b.ws)
    L = nh.workspace_layout(blk.c, T)
    num = int(b.ws[L.num_tiles:L.num_tiles + 4].view(torch.int32).item())
    assert num > 0
    ready = b.ws[L.ready:L.ready + 4 * L.max_tiles].view(torch.int32)
    ready[:num].fill_(-(1 << 24))
    if fmt == "nvfp4":
        nh.forward_nvfp4(blk.c, x, blk.q4["up"], blk.q4["down"], b.ws, b.y_acc)
    else:
        nh.forward(blk.c, x, blk.w_up, blk.w_down, b.ws, b.y_acc)
    torch.cuda.synchronize()
    assert nh.check_device(b.ws) == nh.NH_ERR_TIMEOUT
    assert (ready == 0).all(), "the launch leaves the counters of its tile entries zero"
    y, _, _, _ = run_block(inp, blk)
    assert np.isfinite(y).all()


def test_argument_errors_enqueue_nothing():
    cfg = small_cfg()
    inp = synth.make_inputs(cfg)
    blk = make_block(inp)
    b = blk.buffers(cfg.T)
    x = to_dev(inp.x)
    with pytest.raises(nh.NHMoEError) as e:
        nh.route(blk.c, x, blk.w_router, None, b.topk_idx, b.topk_w, b.ws[:100])
    assert e.value.status == nh.NH_ERR_INVALID_ARG
    with pytest.raises(nh.NHMoEError) as e:
        nh.forward(blk.c, x, blk.w_up, None, b.ws, b.y_acc)
    assert e.value.status == nh.NH_ERR_INVALID_ARG
    torch.cuda.synchronize()
