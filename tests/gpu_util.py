"""Helpers of the GPU parity tests: run the CUDA block on seeded inputs and
compare with the oracle.

Acceptance (the build's parity bar):
  * routing indices bit-exact, in order, except "excused" tokens whose oracle
    selection has a near tie (0 < score gap < 1e-5 at the group or expert
    stage); exact ties (gap == 0) are never excused;
  * routing weights within 1e-5 relative;
  * block output max|err| <= 2e-2 * max|ref| for bf16, <= 1e-4 * max|ref| for
    float32; excused tokens are checked with the oracle under the GPU's routing.
"""
from __future__ import annotations

import os

import numpy as np

import oracle

EXCUSE_GAP = 1e-5
TOL = {"bf16": 2e-2, "f32": 1e-4}
W_RTOL = 1e-5


def threads():
    return max(1, min(32, os.cpu_count() or 1))


def torch_dtype(cfg):
    import torch
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


def to_dev(a, cfg=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.cuda()


def make_block(inp):
    import non_gated_relu_b200 as nh
    return nh.NemotronHMoE(inp.cfg, inp.w_router, inp.w_up, inp.w_down, inp.w_shared_up,
                           inp.w_shared_down, bias=inp.bias, nvfp4=inp.nvfp4,
                           w_latent_fc1=inp.w_latent_fc1, w_latent_fc2=inp.w_latent_fc2)


def run_block(inp, blk=None):
    """Run the whole block on the GPU; returns (y float64, idx, w, block)."""
    import torch
    blk = blk or make_block(inp)
    x = to_dev(inp.x)
    y = blk.forward(x)
    torch.cuda.synchronize()
    rc = blk.check(x.shape[0])
    assert rc == 0, f"device status {rc}"
    b = blk.buffers(x.shape[0])
    return (y.float().cpu().numpy().astype(np.float64), b.topk_idx.cpu().numpy(),
            b.topk_w.cpu().numpy(), blk)


def excused_mask(gg, ge):
    return ((gg > 0) & (gg < EXCUSE_GAP)) | ((ge > 0) & (ge < EXCUSE_GAP))


def check_routing(cfg, x, wr, idx_gpu, w_gpu, bias=None, group_score=0, tie_tokens=None):
    """Compare GPU routing with the oracle; returns (excused mask, oracle idx, oracle w)."""
    o_idx, o_w, gg, ge = oracle.route_parallel(cfg, x, wr, bias, threads=threads(),
                                               group_score=group_score)
    exc = excused_mask(gg, ge)
    if tie_tokens is not None:
        assert not exc[tie_tokens].any(), "exactly tied tokens must never be excused"
    bad = (idx_gpu != o_idx).any(axis=1) & ~exc
    assert not bad.any(), (f"{int(bad.sum())} tokens routed differently, first "
                           f"{np.nonzero(bad)[0][:5]}: gpu {idx_gpu[bad][:3]} oracle {o_idx[bad][:3]}")
    ok = ~exc
    rel = np.abs(w_gpu[ok] - o_w[ok]) / np.abs(o_w[ok])
    assert rel.size == 0 or rel.max() <= W_RTOL, f"topk_w rel err {rel.max():.3g}"
    return exc, o_idx, o_w


def check_output(inp, y_gpu, idx_gpu, w_gpu, tokens, excused):
    """Compare y on `tokens` with the oracle (own routing; GPU routing for excused)."""
    cfg = inp.cfg
    tokens = np.asarray(tokens, np.int64)
    exc_t = tokens[excused[tokens]]
    ok_t = tokens[~excused[tokens]]
    ref = np.zeros((len(tokens), cfg.H))
    order = {t: i for i, t in enumerate(tokens)}
    if len(ok_t):
        y, _, _ = oracle.forward_parallel(inp, tokens=ok_t, threads=threads())
        for i, t in enumerate(ok_t):
            ref[order[t]] = y[i]
    if len(exc_t):
        y, _, _ = oracle.forward_parallel(inp, tokens=exc_t, override_idx=idx_gpu[exc_t],
                                          override_w=w_gpu[exc_t].astype(np.float64),
                                          threads=threads())
        for i, t in enumerate(exc_t):
            ref[order[t]] = y[i]
    got = y_gpu[tokens]
    err = np.abs(got - ref).max()
    scale = np.abs(ref).max()
    tol = TOL[cfg.dtype]
    assert np.isfinite(got).all(), "non-finite output"
    assert err <= tol * scale, f"max|err| {err:.4g} > {tol} * max|ref| {scale:.4g}"
    return err / scale


def assert_same_up_to_sum_order(a, b, dtype):
    """Two runs of the block on the same input: equal up to the order of the
    float32 atomic adds of the combine.  The float32 sums differ by a few
    float32 roundings of the largest term; after the output rounding that is
    at most one ulp of the output type per element (2^-7 relative for bf16),
    plus an absolute float32-level term for sums that cancel to near zero."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    scale = np.abs(b).max()
    rel = 2.0 ** -7 if dtype == "bf16" else 2.0 ** -20
    bound = rel * np.maximum(np.abs(a), np.abs(b)) + 1e-5 * scale
    bad = np.abs(a - b) > bound
    assert not bad.any(), (f"{int(bad.sum())} elements differ beyond the summation-order bound, "
                           f"max |diff| {np.abs(a - b).max():.3g}")


def tile_tokens(blk, T):
    """Tokens that put every tile of the GPU's tile table under test.

    Reads the tile table (expert, first row, rows, kind) and perm_token from
    the block's workspace after a call.  A full 256-row tile (kind 0) is
    computed by a CTA pair, each CTA owning 128 rows: one token from each
    half.  An expert's partial last tile (kind 1, computed swapped), and a
    partial tile attached to a full one (kind 2), give their first and last
    rows.  Returns (tokens, number of tiles, number of kind-1 and kind-2
    tiles)."""
    import non_gated_relu_b200 as nh
    b = blk.buffers(T)
    lay = nh.workspace_layout(blk.c_exp, T)
    ws = b.ws.cpu().numpy()
    n_tiles = int(ws[lay.num_tiles:lay.num_tiles + 4].view(np.int32)[0])
    tiles = ws[lay.tiles:lay.tiles + 16 * n_tiles].view(np.int32).reshape(n_tiles, 4)
    rows = T * blk.k
    perm_token = ws[lay.perm_token:lay.perm_token + 4 * rows].view(np.int32)
    picks = []
    for e, r0, nr, kind in tiles:
        if kind in (0, 2):
            picks += [r0 + 64, r0 + 128 + 63]
            if kind == 2:            # the attached partial tile's first and last rows
                picks += [r0 + 256, r0 + nr - 1]
        else:
            picks += [r0, r0 + nr - 1]
    return (np.unique(perm_token[np.asarray(picks, np.int64)]).astype(np.int64), n_tiles,
            int((tiles[:, 3] >= 1).sum()))


def sample_tokens(T, n, seed, extra=()):
    rng = np.random.default_rng(seed)
    base = rng.choice(T, size=min(n, T), replace=False)
    return np.unique(np.concatenate([base, np.asarray(list(extra), np.int64),
                                     [0, T - 1]])).astype(np.int64)
