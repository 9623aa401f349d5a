"""nh_moe_route_noalloc: the router for callers that cannot allocate.

Some callers cannot give the library a workspace (a serving memory pool that
owns the whole device, a plugin host that passes no scratch buffer and may
not call cudaMalloc).  For them the library keeps the router's scratch in a
fixed array of its own.  This test calls that entry point through the C ABI
twice in a row and checks both results against nh_moe_route, the entry point
with a caller workspace, within the routing tolerance of the other GPU tests
(indices identical, weights within 1e-5 relative).  It runs last (file
name) and works alone in a fresh process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import non_gated_relu_b200 as nh  # noqa: E402

CASES = {
    "decode_30b_layer": dict(T=8),
    "max_tokens": dict(T=32, n_routed_experts=256, n_group=8, topk_group=2,
                       num_experts_per_tok=8, hidden_size=1024, seed=21),
}


def _cfg(**kw):
    return synth.CONFIGS["decode_bf16_t8"].replace(**kw)


@pytest.mark.parametrize("case", sorted(CASES))
def test_noalloc_router_matches_workspace_router(case):
    cfg = _cfg(**CASES[case])
    x_np, wr_np, _, _, _ = synth.make_router_and_x(cfg)
    dev = torch.device("cuda", 0)
    x = torch.from_numpy(x_np).view(torch.bfloat16).to(dev)
    wr = torch.from_numpy(wr_np).to(dev)
    T, k = cfg.T, cfg.k
    lib = nh.load()
    c = nh.config_from(cfg)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    P = ctypes.c_void_p

    ws = torch.empty(nh.workspace_size(c, T), dtype=torch.uint8, device=dev)
    ref_i = torch.empty((T, k), dtype=torch.int32, device=dev)
    ref_w = torch.empty((T, k), dtype=torch.float32, device=dev)
    rc = lib.nh_moe_route(ctypes.byref(c), T, P(x.data_ptr()), P(wr.data_ptr()), None,
                          P(ref_i.data_ptr()), P(ref_w.data_ptr()), P(ws.data_ptr()),
                          ws.numel(), stream)
    assert rc == nh.NH_OK, lib.nh_last_error()

    for call in range(2):
        out_i = torch.full((T, k), -1, dtype=torch.int32, device=dev)
        out_w = torch.zeros((T, k), dtype=torch.float32, device=dev)
        rc = lib.nh_moe_route_noalloc(ctypes.byref(c), T, P(x.data_ptr()), P(wr.data_ptr()),
                                      None, P(out_i.data_ptr()), P(out_w.data_ptr()), stream)
        assert rc == nh.NH_OK, lib.nh_last_error()
        torch.cuda.synchronize(dev)
        np.testing.assert_array_equal(out_i.cpu().numpy(), ref_i.cpu().numpy(),
                                      err_msg=f"call {call}")
        np.testing.assert_allclose(out_w.cpu().numpy(), ref_w.cpu().numpy(), rtol=1e-5, atol=0,
                                   err_msg=f"call {call}")


def test_noalloc_router_rejects_sizes_beyond_its_scratch():
    lib = nh.load()
    P = ctypes.c_void_p
    c = nh.config_from(_cfg(T=33))
    rc = lib.nh_moe_route_noalloc(ctypes.byref(c), 33, P(256), P(256), None, P(256), P(256),
                                  None)
    assert rc == nh.NH_ERR_INVALID_ARG
    assert b"at most 32 tokens" in lib.nh_last_error()
