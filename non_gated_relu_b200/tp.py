"""Tensor-parallel Nemotron-H MoE block: one shard of the expert widths per
GPU, one all-reduce of the block output.

Sharding follows the NemotronHMoE branch of NemotronHShardingStrategy in the
exo commit "Add support for Nemotron sharding"
(src/exo/worker/engines/mlx/auto_parallel.py) and its ShardedMoE wrapper:
  * routed ``fc1`` (up projection, W_up [E, I, H]) and the shared
    ``up_proj`` (W_su [S, H]) are split over their output features;
  * routed ``fc2`` (down projection, W_down [E, H, I]) and the shared
    ``down_proj`` (W_sd [H, S]) are split over their input features;
  * the router (``gate``) is replicated, so every rank routes every token the
    same way;
  * the block output is summed over the ranks by one all-reduce.
relu^2 acts feature by feature, so rank r's slice of I (and of S) gives an
exact part of every output row: y = sum_r y_r.

Layout choice of this library: I and S are split in blocks of 64 features
(the K tile of the expert GEMMs), rank r taking blocks
[r * nb // world, (r + 1) * nb // world).  Shares differ by at most one
block when 64 * world does not divide I (Nemotron-H's I = 1856 is 29
blocks).  Each rank adds its own contributions into its float32
accumulator y_acc without rounding; the all-reduce sums those in float32 and
nh_moe_finalize rounds the sum once, as the unsharded block does.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Tuple

import numpy as np
import torch

from . import NH_WEIGHTS_NVFP4, config_from, finalize
from .block import NemotronHMoE

BLOCK = 64


def shard_range(n: int, world: int, rank: int, block: int = BLOCK) -> Tuple[int, int]:
    """[start, stop) of rank's share of n features, in whole blocks."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if n % block:
        raise ValueError(f"{n} features do not split into blocks of {block}")
    nb = n // block
    if nb < world:
        raise ValueError(f"{n} features ({nb} blocks of {block}) cannot feed {world} ranks")
    return (rank * nb // world) * block, ((rank + 1) * nb // world) * block


def _replace(cfg, **kw):
    return cfg.replace(**kw) if hasattr(cfg, "replace") else dataclasses.replace(cfg, **kw)


def shard_config(cfg, world: int, rank: int):
    """The config a rank runs: its shares of I and S (S stays 0 without a shared expert)."""
    i0, i1 = shard_range(cfg.moe_intermediate_size, world, rank)
    kw = dict(moe_intermediate_size=i1 - i0)
    if cfg.n_shared_experts:
        s0, s1 = shard_range(cfg.moe_shared_expert_intermediate_size, world, rank)
        kw["moe_shared_expert_intermediate_size"] = s1 - s0
    return _replace(cfg, **kw)


def _contig(a):
    return np.ascontiguousarray(a) if isinstance(a, np.ndarray) else a.contiguous()


def shard_weights(cfg, world: int, rank: int, w_up, w_down, w_shared_up=None,
                  w_shared_down=None):
    """Rank's slices of dense weights (numpy or torch, Linear layout)."""
    i0, i1 = shard_range(cfg.moe_intermediate_size, world, rank)
    up = _contig(w_up[:, i0:i1, :])
    down = _contig(w_down[:, :, i0:i1])
    su = sd = None
    if cfg.n_shared_experts and w_shared_up is not None:
        s0, s1 = shard_range(cfg.moe_shared_expert_intermediate_size, world, rank)
        su = _contig(w_shared_up[s0:s1, :])
        sd = _contig(w_shared_down[:, s0:s1])
    return up, down, su, sd


def nvfp4_scale_pitch(cols: int) -> int:
    """Bytes per row of an NVFP4 scale array: ceil(cols / 16) rounded up to 16."""
    return ((cols // 16 + 15) // 16) * 16


def _slice_nvfp4(q, start: int, stop: int, over_inputs: bool):
    """Features [start, stop) of a stacked NVFP4 weight (codes, scales, global).
    over_inputs: the slice runs over the columns (input features), so the codes
    are cut at start / 2 and the scale bytes at start / 16 and re-padded."""
    codes, scales, glob = q
    if not over_inputs:
        return _contig(codes[:, start:stop, :]), _contig(scales[:, start:stop, :]), glob
    c = _contig(codes[:, :, start // 2: stop // 2])
    groups = (stop - start) // 16
    pitch = nvfp4_scale_pitch(stop - start)
    src = scales[:, :, start // 16: start // 16 + groups]
    if isinstance(scales, np.ndarray):
        s = np.zeros(scales.shape[:2] + (pitch,), np.uint8)
    else:
        s = torch.zeros(tuple(scales.shape[:2]) + (pitch,), dtype=scales.dtype,
                        device=scales.device)
    s[:, :, :groups] = src
    return c, s, glob


def shard_nvfp4(cfg, world: int, rank: int, q: dict) -> dict:
    """Rank's slices of NVFP4 weights {"up", "down", "shared_up", "shared_down"}."""
    i0, i1 = shard_range(cfg.moe_intermediate_size, world, rank)
    out = {"up": _slice_nvfp4(q["up"], i0, i1, False),
           "down": _slice_nvfp4(q["down"], i0, i1, True)}
    if cfg.n_shared_experts and "shared_up" in q:
        s0, s1 = shard_range(cfg.moe_shared_expert_intermediate_size, world, rank)
        out["shared_up"] = _slice_nvfp4(q["shared_up"], s0, s1, False)
        out["shared_down"] = _slice_nvfp4(q["shared_down"], s0, s1, True)
    return out


def all_reduce_sum(y: torch.Tensor, group=None) -> torch.Tensor:
    """Sum y over the ranks of `group` in place (one collective; a no-op for
    one rank or without an initialised process group)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
    return y


class TPNemotronHMoE:
    """The block on one rank of a tensor-parallel group.

    Takes the FULL weights (host numpy / torch, as NemotronHMoE) and keeps
    this rank's shard on the device.  ``forward(x)`` runs the whole path on
    the shard, all-reduces the float32 partial output over ``group`` and
    rounds it once into y [T, H].
    """

    def __init__(self, cfg, w_router, w_up=None, w_down=None, w_shared_up=None,
                 w_shared_down=None, bias=None, nvfp4=None, group=None,
                 world: Optional[int] = None, rank: Optional[int] = None, device=None):
        import torch.distributed as dist
        dist_on = dist.is_available() and dist.is_initialized()
        self.world = world if world is not None else (dist.get_world_size(group) if dist_on else 1)
        self.rank = rank if rank is not None else (dist.get_rank(group) if dist_on else 0)
        self.group = group
        self.cfg = cfg
        if getattr(cfg, "latent_size", 0):
            raise NotImplementedError("tensor parallelism of a latent block is not built")
        self.cfg_rank = shard_config(cfg, self.world, self.rank)
        q = None
        if config_from(cfg).weight_format == NH_WEIGHTS_NVFP4:
            q = shard_nvfp4(cfg, self.world, self.rank, nvfp4)
            up = down = su = sd = None
        else:
            up, down, su, sd = shard_weights(cfg, self.world, self.rank, w_up, w_down,
                                             w_shared_up, w_shared_down)
        self.block = NemotronHMoE(self.cfg_rank, w_router, up, down, su, sd, bias=bias,
                                  device=device, nvfp4=q)
        self.c_full = config_from(cfg)
        self._y = {}

    def partial(self, x: torch.Tensor) -> torch.Tensor:
        """This rank's float32 contribution to y (no collective)."""
        return self.block.forward(x, partial=True)

    def output(self, y_f32: torch.Tensor) -> torch.Tensor:
        """y = dtype(y_f32) into this rank's output buffer (the one rounding)."""
        T = y_f32.shape[0]
        y = self._y.get(T)
        if y is None:
            y = torch.empty((T, self.block.H), dtype=self.block.dtype, device=self.block.device)
            self._y[T] = y
        finalize(self.c_full, T, y_f32, y, stream=torch.cuda.current_stream(self.block.device))
        return y

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        y32 = self.partial(x)
        all_reduce_sum(y32, self.group)
        return self.output(y32)

    __call__ = forward
