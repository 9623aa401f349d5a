"""GPU permute against the oracle's stable counting sort, bit-exact.

Checks, for the single-block path (T <= 256), the multi-kernel path and the
fused decode router+permute: counts, offsets, perm_token, perm_w, inv_row
equal oracle.permute of the GPU's own routing; x_perm rows equal x rows; the
tile table covers every expert's rows exactly once in order, with tiles no
taller than the plan's tile height and the partial-tile kind flag set as
documented (kind 1: an expert's partial last tile; kind 2: a full tile with
an attached partial tile of at most 64 rows).
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import non_gated_relu_b200 as nh  # noqa: E402


def region(ws, off, n, dtype):
    b = ws[off: off + n * np.dtype(dtype).itemsize].cpu().numpy()
    return b.view(dtype)


def check_permute(cfg, x_np, idx, w, ws, lay, x_dev):
    E, k, T = cfg.E, cfg.k, cfg.T
    ref = oracle.permute(idx, w, E)
    rows = T * k
    np.testing.assert_array_equal(region(ws, lay.counts, E, np.int32), ref["counts"])
    np.testing.assert_array_equal(region(ws, lay.offsets, E + 1, np.int32), ref["offsets"])
    np.testing.assert_array_equal(region(ws, lay.perm_token, rows, np.int32), ref["perm_token"])
    np.testing.assert_array_equal(region(ws, lay.perm_w, rows, np.float32),
                                  ref["perm_w"].astype(np.float32))
    np.testing.assert_array_equal(region(ws, lay.inv_row, rows, np.int32).reshape(T, k),
                                  ref["inv_row"])
    elem = np.uint16 if cfg.dtype == "bf16" else np.float32
    if not lay.x_direct:   # the decode orientation reads x directly (no x_perm)
        xp = region(ws, lay.x_perm, rows * cfg.H, elem).reshape(rows, cfg.H)
        np.testing.assert_array_equal(xp, x_np[ref["perm_token"]])
    nt = int(region(ws, lay.num_tiles, 1, np.int32)[0])
    tiles = region(ws, lay.tiles, nt * 4, np.int32).reshape(nt, 4)
    covered = np.zeros(rows, np.int32)
    pair = lay.tile_rows == 256
    for e_, r0, n, kind in tiles:
        # CTA-pair tiles: a partial tile of at most 64 rows rides on the
        # expert's last full tile (kind 2); a larger one is its own (kind 1)
        assert 1 <= n <= lay.tile_rows + (64 if pair else 0)
        assert ref["offsets"][e_] <= r0 and r0 + n <= ref["offsets"][e_ + 1]
        want = 0
        if pair:
            want = 1 if n < 256 else (2 if n > 256 else 0)
        assert kind == want
        if kind == 1:           # a small partial tile stands alone only without a full one
            assert n > 64 or ref["counts"][e_] < 256
        if kind == 2:   # the expert's last tile
            assert r0 + n == ref["offsets"][e_ + 1]
        covered[r0:r0 + n] += 1
    assert np.all(covered == 1)
    assert np.all(np.diff(tiles[:, 1]) > 0)


CASES = {
    "decode_t8": dict(T=8),
    "t29_swap32": dict(T=29, seed=31),
    "t200_single_block": dict(T=200, seed=32),
    "t1500_multi_chunk": dict(T=1500, seed=33, n_routed_experts=64),
    "t700_top8_e256": dict(T=700, seed=34, n_routed_experts=256, n_group=8, topk_group=2,
                           num_experts_per_tok=8),
    # few experts: several pair tiles per expert, partial tiles attached or not
    "t1100_e8": dict(T=1100, seed=35, n_routed_experts=8, n_group=2, topk_group=1,
                     num_experts_per_tok=2),
    "t1300_e8": dict(T=1300, seed=36, n_routed_experts=8, n_group=2, topk_group=1,
                     num_experts_per_tok=2),
}


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("fused", [False, True])
def test_permute_matches_counting_sort(case, fused):
    cfg = synth.CONFIGS["decode_bf16_t8"].replace(hidden_size=512, **CASES[case])
    x_np, wr_np, _, _, _ = synth.make_router_and_x(cfg)
    x = to_dev(x_np)
    wr = torch.from_numpy(wr_np).cuda()
    c = nh.config_from(cfg)
    ws = torch.empty(nh.workspace_size(c, cfg.T), dtype=torch.uint8, device="cuda")
    lay = nh.workspace_layout(c, cfg.T)
    ti = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    tw = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device="cuda")
    if fused:
        nh.route_permute(c, x, wr, None, ti, tw, ws)
    else:
        nh.route(c, x, wr, None, ti, tw, ws)
        nh.permute(c, x, ti, tw, ws)
    assert nh.check_device(ws) == 0
    check_permute(cfg, x_np, ti.cpu().numpy(), tw.cpu().numpy(), ws, lay, x)


def test_fused_and_separate_routing_agree():
    cfg = synth.CONFIGS["decode_bf16_t8"]
    x_np, wr_np, _, _, _ = synth.make_router_and_x(cfg)
    x, wr = to_dev(x_np), torch.from_numpy(wr_np).cuda()
    c = nh.config_from(cfg)
    outs = []
    for fused in (False, True):
        ws = torch.empty(nh.workspace_size(c, cfg.T), dtype=torch.uint8, device="cuda")
        ti = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
        tw = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device="cuda")
        if fused:
            nh.route_permute(c, x, wr, None, ti, tw, ws)
        else:
            nh.route(c, x, wr, None, ti, tw, ws)
            nh.permute(c, x, ti, tw, ws)
        torch.cuda.synchronize()
        outs.append((ti.cpu().numpy(), tw.cpu().numpy()))
    np.testing.assert_array_equal(outs[0][0], outs[1][0])
    # the two router kernels reduce the logits in different orders
    np.testing.assert_allclose(outs[0][1], outs[1][1], rtol=1e-6, atol=0)
