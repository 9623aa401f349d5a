"""Seeded synthetic inputs for the Nemotron-H non-gated MoE block.

This module is shared by the CPU oracle, the tests and the benchmark.  It
holds only workload definitions and random-number recipes: no step of the
MoE arithmetic (no routing, no matmul, no activation) lives here.

Workloads follow the MoE layer printed on the pages:
  * baseRT issue #46, "Architecture (config.json)": 128 routed experts, 6 per
    token, n_groups=8, topk_group=1, routed_scaling_factor=2.5,
    norm_topk_prob, 1 shared expert 3712 wide, relu2, no gate_proj;
  * auto-round PR #1712, the unfused-experts log: 128 x
    (up_proj Linear(2688->1856), down_proj Linear(1856->2688)), bias=False.

Every tensor is drawn from its own PCG64 stream,
``numpy.random.default_rng([seed, tensor_id, sub])`` (``sub`` = expert id for
the stacked expert weights), as float32 standard normals times the stated
standard deviation, then rounded to the storage dtype (bf16: round to
nearest even on the float32 bits).  Independent streams let any tensor (or
any one expert) be regenerated without drawing the others.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np

# tensor ids of the independent streams
_X, _WR, _WUP, _WDOWN, _WSU, _WSD, _SKEW, _TIE, _BIAS = range(1, 10)


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    """Shape of one MoE block plus the token count of the workload.

    Field names are the config.json names of the Nemotron-H model (MLX
    ``ModelArgs`` in the exo commit "Add support for Nemotron sharding").
    ``n_group`` is the router's group count (the pages' MoE summary also
    spells it "n_groups", which in ``ModelArgs`` is the Mamba-2 field).
    """
    name: str
    T: int
    hidden_size: int
    n_routed_experts: int
    n_group: int
    topk_group: int
    num_experts_per_tok: int
    moe_intermediate_size: int
    moe_shared_expert_intermediate_size: int
    n_shared_experts: int = 1
    norm_topk_prob: bool = True
    routed_scaling_factor: float = 2.5
    dtype: str = "bf16"          # activations and expert weights; router is fp32
    seed: int = 0
    x_std: float = 1.0
    w_std: float = 0.02
    wr_std: float = 0.02         # router weight standard deviation
    skew_hot_groups: int = 0     # >0: skewed routing (hot experts, bias feature)
    skew_hot_per_group: int = 0
    tie_fraction: float = 0.0    # fraction of tokens built to tie exactly
    tie_columns: int = 0

    # short aliases used by the kernels' notation
    @property
    def H(self): return self.hidden_size
    @property
    def E(self): return self.n_routed_experts
    @property
    def G(self): return self.n_group
    @property
    def tg(self): return self.topk_group
    @property
    def k(self): return self.num_experts_per_tok
    @property
    def I(self): return self.moe_intermediate_size
    @property
    def S(self): return self.moe_shared_expert_intermediate_size

    def replace(self, **kw) -> "MoEConfig":
        return dataclasses.replace(self, **kw)

    def flops_per_token(self) -> int:
        """Algorithmic flops per token: router GEMV + k routed MLPs + shared MLP."""
        f = 2 * self.H * self.E + self.k * 4 * self.H * self.I
        if self.n_shared_experts:
            f += 4 * self.H * self.S
        return f


# The five workloads of the build.  Shapes 2-4 are the 30B-A3B layer.
CONFIGS = {
    "tiny_f32_t64": MoEConfig(
        "tiny_f32_t64", T=64, hidden_size=256, n_routed_experts=16, n_group=4,
        topk_group=1, num_experts_per_tok=2, moe_intermediate_size=128,
        moe_shared_expert_intermediate_size=256, dtype="f32", seed=0,
        wr_std=0.05),
    "decode_bf16_t8": MoEConfig(
        "decode_bf16_t8", T=8, hidden_size=2688, n_routed_experts=128, n_group=8,
        topk_group=1, num_experts_per_tok=6, moe_intermediate_size=1856,
        moe_shared_expert_intermediate_size=3712, seed=1),
    "prefill_skewed_bf16_t2048": MoEConfig(
        "prefill_skewed_bf16_t2048", T=2048, hidden_size=2688, n_routed_experts=128,
        n_group=8, topk_group=1, num_experts_per_tok=6, moe_intermediate_size=1856,
        moe_shared_expert_intermediate_size=3712, seed=2,
        skew_hot_groups=4, skew_hot_per_group=2),
    "prefill_bf16_t16384": MoEConfig(
        "prefill_bf16_t16384", T=16384, hidden_size=2688, n_routed_experts=128,
        n_group=8, topk_group=1, num_experts_per_tok=6, moe_intermediate_size=1856,
        moe_shared_expert_intermediate_size=3712, seed=3,
        wr_std=float(1.0 / np.sqrt(2688))),
    "stress_bf16_t4096": MoEConfig(
        "stress_bf16_t4096", T=4096, hidden_size=4096, n_routed_experts=256, n_group=8,
        topk_group=2, num_experts_per_tok=8, moe_intermediate_size=2048,
        moe_shared_expert_intermediate_size=4096, seed=4,
        tie_fraction=0.05, tie_columns=8),
}

CONFIG_ORDER = list(CONFIGS)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return the bits as uint16."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u >> np.uint32(16)) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r >>= np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 exactly."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal(seed: int, tid: int, sub: int, shape, std: float) -> np.ndarray:
    rng = np.random.default_rng([seed, tid, sub])
    a = rng.standard_normal(int(np.prod(shape)), dtype=np.float32).reshape(shape)
    if std != 1.0:
        a *= np.float32(std)
    return a


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(a) if dtype == "bf16" else np.ascontiguousarray(a, np.float32)


@dataclasses.dataclass
class MoEInputs:
    """Host arrays of one workload.  bf16 tensors are uint16 bit patterns.

    Layouts (row-major, PyTorch ``Linear`` weight layout ``[out, in]``):
      x [T, H]; w_router [E, H] float32; w_up [E, I, H]; w_down [E, H, I];
      w_shared_up [S, H]; w_shared_down [H, S]; bias [E] float32 or None.
    """
    cfg: MoEConfig
    x: np.ndarray
    w_router: np.ndarray
    w_up: np.ndarray
    w_down: np.ndarray
    w_shared_up: Optional[np.ndarray]
    w_shared_down: Optional[np.ndarray]
    bias: Optional[np.ndarray] = None
    hot_experts: Optional[np.ndarray] = None
    tie_tokens: Optional[np.ndarray] = None
    tie_cols: Optional[np.ndarray] = None
    skew_b: Optional[float] = None


def default_threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def make_router_and_x(cfg: MoEConfig, skew_b: Optional[float] = None):
    """Draw x and the router weight (and the skew / tie structure) only.

    Returns (x, w_router, hot_experts, tie_tokens, tie_cols).
    """
    T, H, E = cfg.T, cfg.H, cfg.E
    x = _normal(cfg.seed, _X, 0, (T, H), cfg.x_std)
    wr = _normal(cfg.seed, _WR, 0, (E, H), cfg.wr_std)
    hot = ties = tcols = None
    if cfg.skew_hot_groups:
        rng = np.random.default_rng([cfg.seed, _SKEW, 0])
        g = E // cfg.G
        groups = np.sort(rng.choice(cfg.G, size=cfg.skew_hot_groups, replace=False))
        hot = np.sort(np.concatenate([
            q * g + np.sort(rng.choice(g, size=cfg.skew_hot_per_group, replace=False))
            for q in groups])).astype(np.int32)
        # a constant feature routed to the hot experts with weight b
        x[:, H - 1] = 1.0
        wr[:, H - 1] = 0.0
        wr[hot, H - 1] = np.float32(0.0 if skew_b is None else skew_b)
    x = _store(x, cfg.dtype)
    if cfg.tie_fraction > 0:
        rng = np.random.default_rng([cfg.seed, _TIE, 0])
        n_tie = int(round(cfg.tie_fraction * T))
        ties = np.sort(rng.choice(T, size=n_tie, replace=False)).astype(np.int64)
        tcols = np.sort(rng.choice(H, size=cfg.tie_columns, replace=False)).astype(np.int64)
        # router column values drawn from {+-2^-5, +-2^-4}: exact products
        vals = np.array([2.0 ** -5, -(2.0 ** -5), 2.0 ** -4, -(2.0 ** -4)], np.float32)
        wr[:, tcols] = vals[rng.integers(0, 4, size=(E, cfg.tie_columns))]
        s = rng.standard_normal(n_tie, dtype=np.float32)
        j = tcols[rng.integers(0, cfg.tie_columns, size=n_tie)]
        s_st = _store(s, cfg.dtype)
        zero = _store(np.zeros(1, np.float32), cfg.dtype)[0]
        x[ties, :] = zero
        x[ties, j] = s_st
    return x, np.ascontiguousarray(wr, np.float32), hot, ties, tcols


def make_expert(cfg: MoEConfig, e: int):
    """(w_up[e] [I, H], w_down[e] [H, I]) of routed expert e, in the storage dtype."""
    up = _store(_normal(cfg.seed, _WUP, e, (cfg.I, cfg.H), cfg.w_std), cfg.dtype)
    down = _store(_normal(cfg.seed, _WDOWN, e, (cfg.H, cfg.I), cfg.w_std), cfg.dtype)
    return up, down


def make_inputs(cfg: MoEConfig, skew_b: Optional[float] = None,
                threads: Optional[int] = None, with_bias: bool = False) -> MoEInputs:
    """All inputs of a workload (expert weights drawn in parallel threads)."""
    x, wr, hot, ties, tcols = make_router_and_x(cfg, skew_b)
    sdt = np.uint16 if cfg.dtype == "bf16" else np.float32
    w_up = np.empty((cfg.E, cfg.I, cfg.H), sdt)
    w_down = np.empty((cfg.E, cfg.H, cfg.I), sdt)

    def fill(e):
        w_up[e], w_down[e] = make_expert(cfg, e)

    with ThreadPoolExecutor(threads or default_threads()) as ex:
        list(ex.map(fill, range(cfg.E)))
    wsu = wsd = None
    if cfg.n_shared_experts:
        wsu = _store(_normal(cfg.seed, _WSU, 0, (cfg.S, cfg.H), cfg.w_std), cfg.dtype)
        wsd = _store(_normal(cfg.seed, _WSD, 0, (cfg.H, cfg.S), cfg.w_std), cfg.dtype)
    bias = None
    if with_bias:
        bias = _normal(cfg.seed, _BIAS, 0, (cfg.E,), 0.1).astype(np.float32)
    return MoEInputs(cfg, x, wr, w_up, w_down, wsu, wsd, bias, hot, ties, tcols, skew_b)


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 view of a stored tensor (bf16 bits or float32)."""
    if dtype == "bf16" and a.dtype == np.uint16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, np.float64)
