"""Seeded synthetic inputs for the Nemotron-H non-gated MoE block.

This module is shared by the CPU oracle, the tests and the benchmark.  It
holds only workload definitions and random-number recipes: no step of the
MoE arithmetic (no routing, no matmul, no activation) lives here.

Workloads follow the Nemotron-H MoE layer as these sources give it:
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
_X, _WR, _WUP, _WDOWN, _WSU, _WSD, _SKEW, _TIE, _BIAS, _WL1, _WL2 = range(1, 12)


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    """Shape of one MoE block plus the token count of the workload.

    Field names are the config.json names of the Nemotron-H model (MLX
    ``ModelArgs`` in the exo commit "Add support for Nemotron sharding").
    ``n_group`` is the router's group count (the baseRT MoE summary also
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
    weight_format: str = "native"  # expert / shared weights: "native" (= dtype) or "nvfp4"
    seed: int = 0
    x_std: float = 1.0
    w_std: float = 0.02
    wr_std: float = 0.02         # router weight standard deviation
    skew_hot_groups: int = 0     # >0: skewed routing (hot experts, bias feature)
    skew_hot_per_group: int = 0
    tie_fraction: float = 0.0    # fraction of tokens built to tie exactly
    tie_columns: int = 0
    latent_size: int = 0         # >0: routed experts in this width between
                                 # fc1_latent_proj [L, H] and fc2_latent_proj [H, L]

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
    @property
    def L(self): return self.latent_size
    @property
    def HE(self):
        """Width of the routed experts' input and output (hidden or latent)."""
        return self.latent_size or self.hidden_size

    def replace(self, **kw) -> "MoEConfig":
        return dataclasses.replace(self, **kw)

    def flops_per_token(self) -> int:
        """Algorithmic flops per token: router GEMV + k routed MLPs + shared MLP."""
        f = 2 * self.H * self.E + self.k * 4 * self.HE * self.I
        if self.n_shared_experts:
            f += 4 * self.H * self.S
        if self.latent_size:
            f += 4 * self.H * self.latent_size
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
    "decode_nvfp4_t8": MoEConfig(
        "decode_nvfp4_t8", T=8, hidden_size=2688, n_routed_experts=128, n_group=8,
        topk_group=1, num_experts_per_tok=6, moe_intermediate_size=1856,
        moe_shared_expert_intermediate_size=3712, seed=5, weight_format="nvfp4"),
    "stress_bf16_t4096": MoEConfig(
        "stress_bf16_t4096", T=4096, hidden_size=4096, n_routed_experts=256, n_group=8,
        topk_group=2, num_experts_per_tok=8, moe_intermediate_size=2048,
        moe_shared_expert_intermediate_size=4096, seed=4,
        tie_fraction=0.05, tie_columns=8),
    # latent projections around the routed experts (width 1024), decode shape
    "decode_latent_bf16_t8": MoEConfig(
        "decode_latent_bf16_t8", T=8, hidden_size=2688, n_routed_experts=128, n_group=8,
        topk_group=1, num_experts_per_tok=6, moe_intermediate_size=1856,
        moe_shared_expert_intermediate_size=3712, seed=6, latent_size=1024),
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


# ---------------------------------------------------------------------------
# NVFP4 weight encoding (input generation: the weights of an "nvfp4" workload
# are drawn as float32, then encoded; the oracle and the CUDA library each
# decode them with their own code)
# ---------------------------------------------------------------------------
_E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
# decision boundaries between neighbouring magnitudes; a value on a boundary
# goes to the magnitude with an even code (round to nearest even)
_E2M1_EDGE = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
_E2M1_TIE_UP = np.array([False, True, False, True, False, True, False])


def _e4m3_positive_table():
    codes = np.arange(0, 0x7F, dtype=np.int64)             # 0x7F is NaN
    e, m = codes >> 3, codes & 7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1 + m / 8.0) * 2.0 ** (e - 7))
    return codes, val


_E4M3_CODES, _E4M3_VALS = _e4m3_positive_table()


def _e4m3_encode_positive(v):
    """Nearest E4M3 code of non-negative values (ties to even code), saturating at 448."""
    v = np.minimum(np.asarray(v, np.float64), _E4M3_VALS[-1])
    hi = np.clip(np.searchsorted(_E4M3_VALS, v), 1, len(_E4M3_VALS) - 1)
    lo = hi - 1
    dlo, dhi = v - _E4M3_VALS[lo], _E4M3_VALS[hi] - v
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (_E4M3_CODES[hi] % 2 == 0))
    return np.where(pick_hi, _E4M3_CODES[hi], _E4M3_CODES[lo]).astype(np.uint8)


def _e2m1_encode(q):
    a = np.abs(q)
    idx = np.searchsorted(_E2M1_EDGE, a, side="left")      # a <= edge -> lower magnitude
    on_edge = np.zeros(a.shape, bool)
    for i, edge in enumerate(_E2M1_EDGE):
        on_edge |= (a == edge) & _E2M1_TIE_UP[i] & (idx == i)
    idx = np.minimum(idx + on_edge, 7)
    sign = (q < 0) & (idx > 0)
    return (idx | (sign.astype(np.int64) << 3)).astype(np.uint8)


def nvfp4_scale_pitch(cols: int) -> int:
    """Bytes per row of scale factors: one per 16 columns, padded to 16 bytes."""
    return ((cols // 16 + 15) // 16) * 16


def quantize_nvfp4(w: np.ndarray):
    """Encode float weights [n_mat, rows, cols] (cols % 16 == 0) as NVFP4.

    Returns (codes uint8 [n_mat, rows, cols/2], scales uint8 [n_mat, rows,
    pitch], global float32 [n_mat]): per matrix a global scale amax/(6*448),
    per 16 columns an E4M3 scale nearest to block_amax/6/global, per element
    the E2M1 code nearest to w / (scale * global) (ties to even)."""
    w = np.asarray(w, np.float32)
    n, r, c = w.shape
    assert c % 16 == 0
    amax = np.abs(w).reshape(n, -1).max(axis=1).astype(np.float64)
    g = np.where(amax > 0, amax / (6.0 * 448.0), 1.0).astype(np.float32)
    blocks = w.reshape(n, r, c // 16, 16).astype(np.float64)
    bmax = np.abs(blocks).max(axis=-1)
    scode = _e4m3_encode_positive(bmax / 6.0 / g[:, None, None].astype(np.float64))
    sval = _E4M3_VALS[scode.astype(np.int64)] * g[:, None, None].astype(np.float64)
    q = np.where(sval[..., None] > 0, blocks / np.where(sval > 0, sval, 1.0)[..., None], 0.0)
    codes = _e2m1_encode(q).reshape(n, r, c)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    pitch = nvfp4_scale_pitch(c)
    scales = np.zeros((n, r, pitch), np.uint8)
    scales[..., : c // 16] = scode
    return packed, scales, g


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
    # NVFP4 workloads: {"up", "down", "shared_up", "shared_down"} ->
    # (codes, scales, global) as returned by quantize_nvfp4
    nvfp4: Optional[dict] = None
    # latent workloads: fc1_latent_proj [L, H], fc2_latent_proj [H, L] (dtype);
    # w_up is then [E, I, L] and w_down [E, L, I]
    w_latent_fc1: Optional[np.ndarray] = None
    w_latent_fc2: Optional[np.ndarray] = None


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
    """(w_up[e] [I, HE], w_down[e] [HE, I]) of routed expert e, in the storage
    dtype (HE = hidden size, or the latent size of a latent workload)."""
    up = _store(_normal(cfg.seed, _WUP, e, (cfg.I, cfg.HE), cfg.w_std), cfg.dtype)
    down = _store(_normal(cfg.seed, _WDOWN, e, (cfg.HE, cfg.I), cfg.w_std), cfg.dtype)
    return up, down


def make_latent(cfg: MoEConfig):
    """(fc1_latent_proj [L, H], fc2_latent_proj [H, L]) in the storage dtype,
    drawn with standard deviations 1/sqrt(H) and 1/sqrt(L) (unit-variance
    latent activations for unit-variance x), or (None, None)."""
    if not cfg.latent_size:
        return None, None
    L, H = cfg.latent_size, cfg.H
    w1 = _store(_normal(cfg.seed, _WL1, 0, (L, H), H ** -0.5), cfg.dtype)
    w2 = _store(_normal(cfg.seed, _WL2, 0, (H, L), L ** -0.5), cfg.dtype)
    return w1, w2


def make_inputs(cfg: MoEConfig, skew_b: Optional[float] = None,
                threads: Optional[int] = None, with_bias: bool = False) -> MoEInputs:
    """All inputs of a workload (expert weights drawn in parallel threads)."""
    x, wr, hot, ties, tcols = make_router_and_x(cfg, skew_b)
    if cfg.weight_format == "nvfp4":
        return _make_nvfp4_inputs(cfg, x, wr, hot, ties, tcols, skew_b, threads, with_bias)
    sdt = np.uint16 if cfg.dtype == "bf16" else np.float32
    w_up = np.empty((cfg.E, cfg.I, cfg.HE), sdt)
    w_down = np.empty((cfg.E, cfg.HE, cfg.I), sdt)

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
    wl1, wl2 = make_latent(cfg)
    return MoEInputs(cfg, x, wr, w_up, w_down, wsu, wsd, bias, hot, ties, tcols, skew_b,
                     w_latent_fc1=wl1, w_latent_fc2=wl2)


def _make_nvfp4_inputs(cfg, x, wr, hot, ties, tcols, skew_b, threads, with_bias):
    """Weights drawn as float32 (same streams as the native format) and encoded
    as NVFP4, one matrix per thread task."""
    E, H, I, S = cfg.E, cfg.HE, cfg.I, cfg.S
    pu, pd = nvfp4_scale_pitch(H), nvfp4_scale_pitch(I)
    up = (np.empty((E, I, H // 2), np.uint8), np.empty((E, I, pu), np.uint8), np.empty(E, np.float32))
    dn = (np.empty((E, H, I // 2), np.uint8), np.empty((E, H, pd), np.uint8), np.empty(E, np.float32))

    def fill(e):
        u = _normal(cfg.seed, _WUP, e, (I, H), cfg.w_std)
        d = _normal(cfg.seed, _WDOWN, e, (H, I), cfg.w_std)
        for dst, w in ((up, u), (dn, d)):
            c, sc, g = quantize_nvfp4(w[None])
            dst[0][e], dst[1][e], dst[2][e] = c[0], sc[0], g[0]

    with ThreadPoolExecutor(threads or default_threads()) as ex:
        list(ex.map(fill, range(E)))
    q = {"up": up, "down": dn}
    if cfg.n_shared_experts:
        Hs = cfg.H
        q["shared_up"] = quantize_nvfp4(_normal(cfg.seed, _WSU, 0, (S, Hs), cfg.w_std)[None])
        q["shared_down"] = quantize_nvfp4(_normal(cfg.seed, _WSD, 0, (Hs, S), cfg.w_std)[None])
    bias = _normal(cfg.seed, _BIAS, 0, (E,), 0.1).astype(np.float32) if with_bias else None
    wl1, wl2 = make_latent(cfg)
    return MoEInputs(cfg, x, wr, None, None, None, None, bias, hot, ties, tcols, skew_b, q,
                     w_latent_fc1=wl1, w_latent_fc2=wl2)


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 view of a stored tensor (bf16 bits or float32)."""
    if dtype == "bf16" and a.dtype == np.uint16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, np.float64)
