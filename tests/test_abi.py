"""C ABI of libnhmoe on the host (no GPU): the library loads, exports every
function include/nh_moe.h declares, and its host-side logic (validation,
workspace plan, argument checks) behaves as documented."""
import ctypes
import os
import re

import pytest

import non_gated_relu_b200 as nh
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


def declared_functions():
    names = []
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(nh_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported():
    lib = nh.load()
    names = declared_functions()
    assert "nh_moe_route" in names and "nh_moe_forward" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared but not exported"
    assert set(nh._EXPORTS) <= set(names)


def test_version_string():
    assert b"sm_100a" in nh.load().nh_version()


@pytest.mark.parametrize("name", synth.CONFIG_ORDER)
def test_workload_configs_validate(name):
    nh.validate(synth.CONFIGS[name])


def test_validation_rejects_bad_configs():
    base = synth.CONFIGS["decode_bf16_t8"]
    bad = [dict(n_group=7), dict(topk_group=9), dict(topk_group=0), dict(num_experts_per_tok=17),
           dict(num_experts_per_tok=0), dict(routed_scaling_factor=float("inf")),
           dict(n_shared_experts=2), dict(hidden_size=0)]
    for kw in bad:
        with pytest.raises(nh.NHMoEError) as e:
            nh.validate(base.replace(**kw))
        assert e.value.status == nh.NH_ERR_INVALID_ARG, kw
    for kw in [dict(hidden_size=2690), dict(moe_intermediate_size=1850),
               dict(n_routed_experts=1024, n_group=8)]:
        with pytest.raises(nh.NHMoEError) as e:
            nh.validate(base.replace(**kw))
        assert e.value.status == nh.NH_ERR_UNSUPPORTED, kw
    # the float32 path takes any size
    nh.validate(base.replace(dtype="f32", hidden_size=2690, moe_intermediate_size=1850))
    # NVFP4 weights need bf16 activations
    with pytest.raises(nh.NHMoEError) as e:
        nh.validate(base.replace(dtype="f32", weight_format="nvfp4"))
    assert e.value.status == nh.NH_ERR_INVALID_ARG
    nh.validate(base.replace(weight_format="nvfp4"))
    # top-2 group score needs two experts per group
    c = nh.config_from(base.replace(n_routed_experts=8, n_group=8, num_experts_per_tok=1))
    c.group_score = 1
    with pytest.raises(nh.NHMoEError):
        nh.validate(c)


@pytest.mark.parametrize("name", synth.CONFIG_ORDER)
def test_workspace_layout(name):
    cfg = synth.CONFIGS[name]
    T = cfg.T
    L = nh.workspace_layout(cfg, T)
    assert L.total_bytes == nh.workspace_size(cfg, T)
    rows = T * cfg.k
    elem = 2 if cfg.dtype == "bf16" else 4
    regions = [("status", 16), ("logits", T * cfg.E * 4),
               ("router_w", cfg.E * 3 * cfg.H * 2 if cfg.dtype == "bf16" else 1),
               ("counts", cfg.E * 4),
               ("offsets", (cfg.E + 1) * 4), ("chunk_counts", L.n_chunks * cfg.E * 4),
               ("perm_token", rows * 4), ("perm_w", rows * 4), ("inv_row", rows * 4),
               ("tiles", L.max_tiles * 16), ("num_tiles", 4), ("x_perm", 0 if L.x_direct else rows * cfg.H * elem),
               ("h", rows * cfg.I * elem), ("ready", L.max_tiles * 4)]
    spans = sorted((getattr(L, n), getattr(L, n) + sz, n) for n, sz in regions)
    for (a0, a1, an), (b0, b1, bn) in zip(spans, spans[1:]):
        assert a1 <= b0, (an, bn)
    assert spans[-1][1] <= L.total_bytes
    assert all(getattr(L, n) % 256 == 0 for n, _ in regions)
    # tile plan: decode-sized T puts weights on the MMA M side
    if cfg.weight_format == "nvfp4":
        assert L.swap_ab == 1 and L.tile_rows in (16, 32, 64)
    elif cfg.dtype == "f32":
        assert L.tile_rows == 64 and L.swap_ab == 0
    elif T <= 64:
        assert L.swap_ab == 1 and L.tile_rows >= T and L.tile_rows % 16 == 0
    else:
        assert L.swap_ab == 0 and L.tile_rows == 256     # CTA-pair tiles
    assert L.max_tiles >= -(-rows // L.tile_rows) + cfg.E - 1


def test_argument_checks_before_any_device_work():
    lib = nh.load()
    c = nh.config_from(synth.CONFIGS["decode_bf16_t8"])
    P = ctypes.c_void_p
    # NULL workspace
    rc = lib.nh_moe_route(ctypes.byref(c), 8, P(16), P(16), None, P(16), P(16), None, 0, None)
    assert rc == nh.NH_ERR_INVALID_ARG and b"ws" in lib.nh_last_error()
    # workspace too small
    rc = lib.nh_moe_permute(ctypes.byref(c), 8, P(16), P(16), P(16), P(256), 10, None)
    assert rc == nh.NH_ERR_INVALID_ARG and b"needed" in lib.nh_last_error()
    # misaligned pointer
    need = nh.workspace_size(c, 8)
    rc = lib.nh_moe_forward(ctypes.byref(c), 8, P(16), P(18), P(16), P(256), need, P(256), None)
    assert rc == nh.NH_ERR_INVALID_ARG and b"aligned" in lib.nh_last_error()
    # the routed combine needs its float32 accumulator
    rc = lib.nh_moe_forward(ctypes.byref(c), 8, P(16), P(16), P(16), P(256), need, None, None)
    assert rc == nh.NH_ERR_INVALID_ARG and b"y_acc" in lib.nh_last_error()
    rc = lib.nh_moe_experts_down(ctypes.byref(c), 8, P(16), P(256), need, P(260), None)
    assert rc == nh.NH_ERR_INVALID_ARG and b"y_acc" in lib.nh_last_error()
    # negative T
    rc = lib.nh_moe_workspace_size(ctypes.byref(c), -1, ctypes.byref(ctypes.c_size_t()))
    assert rc == nh.NH_ERR_INVALID_ARG
    # shared workspace of a config without a shared expert
    c0 = nh.config_from(synth.CONFIGS["decode_bf16_t8"].replace(n_shared_experts=0))
    rc = lib.nh_moe_shared_workspace_size(ctypes.byref(c0), 8, ctypes.byref(ctypes.c_size_t()))
    assert rc == nh.NH_ERR_INVALID_ARG
    # finalize reads the accumulator and writes y
    rc = lib.nh_moe_finalize(ctypes.byref(c), 8, None, P(16), None)
    assert rc == nh.NH_ERR_INVALID_ARG and b"y_acc" in lib.nh_last_error()
    rc = lib.nh_moe_finalize(ctypes.byref(c), 8, P(256), P(264), None)
    assert rc == nh.NH_ERR_INVALID_ARG and b"aligned" in lib.nh_last_error()
    rc = lib.nh_moe_finalize(ctypes.byref(c), -1, P(256), P(256), None)
    assert rc == nh.NH_ERR_INVALID_ARG
    rc = lib.nh_moe_zero_acc(ctypes.byref(c), 8, P(250), None)
    assert rc == nh.NH_ERR_INVALID_ARG and b"aligned" in lib.nh_last_error()
    # zero tokens: nothing to do, no device needed
    assert lib.nh_moe_finalize(ctypes.byref(c), 0, None, None, None) == nh.NH_OK
    assert lib.nh_moe_zero_acc(ctypes.byref(c), 0, None, None) == nh.NH_OK
    # selftest timeout bound
    rc = lib.nh_moe_selftest_timeout(P(256), 0, None)
    assert rc == nh.NH_ERR_INVALID_ARG


def test_zero_tokens_is_a_no_op_plan():
    cfg = synth.CONFIGS["decode_bf16_t8"]
    L = nh.workspace_layout(cfg, 0)
    assert L.total_bytes > 0 and L.n_chunks == 0


def test_latent_config_is_the_expert_width_block():
    cfg = synth.CONFIGS["decode_latent_bf16_t8"]
    e = nh.latent_config(cfg)
    c = nh.config_from(cfg)
    assert (e.hidden_size, e.latent_size, e.n_shared_experts) == (cfg.latent_size, 0, 0)
    for f in ("n_routed_experts", "n_group", "topk_group", "num_experts_per_tok",
              "moe_intermediate_size", "norm_topk_prob", "routed_scaling_factor", "dtype",
              "group_score", "weight_format"):
        assert getattr(e, f) == getattr(c, f), f
    assert nh.latent_workspace_size(cfg, cfg.T) >= 16 * 4
    # a plain block has no expert-width config and no latent workspace
    plain = synth.CONFIGS["decode_bf16_t8"]
    for fn in (lambda: nh.latent_config(plain), lambda: nh.latent_workspace_size(plain, 8)):
        with pytest.raises(nh.NHMoEError) as e:
            fn()
        assert e.value.status == nh.NH_ERR_INVALID_ARG
    # bf16 tiles need a latent width that is a multiple of 64
    with pytest.raises(nh.NHMoEError) as e:
        nh.validate(cfg.replace(latent_size=100))
    assert e.value.status in (nh.NH_ERR_INVALID_ARG, nh.NH_ERR_UNSUPPORTED)
    nh.validate(cfg.replace(dtype="f32", latent_size=100))


def test_next_row_argument_checks_before_any_device_work():
    lib = nh.load()
    P = ctypes.c_void_p
    lat = nh.config_from(synth.CONFIGS["decode_latent_bf16_t8"])
    need = nh.workspace_size(synth.CONFIGS["decode_bf16_t8"], 8)
    # routed-expert calls refuse the full latent config
    for rc in (lib.nh_moe_permute(ctypes.byref(lat), 8, P(256), P(256), P(256), P(256), need, None),
               lib.nh_moe_forward(ctypes.byref(lat), 8, P(256), P(256), P(256), P(256), need,
                                  P(256), None)):
        assert rc == nh.NH_ERR_INVALID_ARG and b"latent_size" in lib.nh_last_error()
    # latent projections: workspace and pointer checks
    rc = lib.nh_moe_latent_in(ctypes.byref(lat), 8, P(256), P(256), P(256), None, 256, None)
    assert rc == nh.NH_ERR_INVALID_ARG and b"ws_latent" in lib.nh_last_error()
    rc = lib.nh_moe_latent_in(ctypes.byref(lat), 8, P(256), P(256), P(256), P(256), 8, None)
    assert rc == nh.NH_ERR_INVALID_ARG and b"needed" in lib.nh_last_error()
    rc = lib.nh_moe_latent_out(ctypes.byref(lat), 8, P(256), P(258), P(256), P(256), 256, None)
    assert rc == nh.NH_ERR_INVALID_ARG and b"aligned" in lib.nh_last_error()
    # NVFP4 entry points: NULL weight descriptors, and the format must match the call
    q4 = nh.config_from(synth.CONFIGS["decode_nvfp4_t8"])
    rc = lib.nh_moe_forward_nvfp4(ctypes.byref(q4), 8, P(256), None, None, P(256), need, P(256),
                                  None)
    assert rc == nh.NH_ERR_INVALID_ARG and b"NULL" in lib.nh_last_error()
    rc = lib.nh_moe_forward(ctypes.byref(q4), 8, P(256), P(256), P(256), P(256),
                            nh.workspace_size(synth.CONFIGS["decode_nvfp4_t8"], 8), P(256), None)
    assert rc == nh.NH_ERR_INVALID_ARG and b"NVFP4" in lib.nh_last_error()
    w = nh.NvFp4Weight(256, 256, 256)
    bf = nh.config_from(synth.CONFIGS["decode_bf16_t8"])
    rc = lib.nh_moe_forward_nvfp4(ctypes.byref(bf), 8, P(256), ctypes.byref(w), ctypes.byref(w),
                                  P(256), need, P(256), None)
    assert rc == nh.NH_ERR_INVALID_ARG and b"native" in lib.nh_last_error()
    rc = lib.nh_moe_forward_nvfp4(ctypes.byref(q4), 8, P(256), ctypes.byref(w), ctypes.byref(w),
                                  P(256), need, None, None)
    assert rc == nh.NH_ERR_INVALID_ARG and b"y_acc" in lib.nh_last_error()
