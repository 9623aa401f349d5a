"""Python binding of libnhmoe, the B200 (sm_100a) Nemotron-H non-gated MoE block.

Argument marshalling only: every step of the block runs in the CUDA kernels
behind the C ABI declared in ``include/nh_moe.h``.  PyTorch supplies device
memory and streams.  There is no CPU fallback: when the library cannot be
built or loaded, or no sm_100 device is present, the calls raise.

Low level (same names as the C ABI, minus the ``nh_moe_`` prefix):
``route``, ``permute``, ``forward``, ``shared``, ``zero_acc``, ``finalize``,
``check_device``, ``workspace_size``, ``workspace_layout``,
``shared_workspace_size``, ``validate``, ``selftest_timeout``.

Block level: :class:`NemotronHMoE` (``block.py``) holds the weights and
buffers and runs one block call on two streams (optionally as a CUDA graph).
"""
from __future__ import annotations

import ctypes
import os
import threading

from . import build as _build

__all__ = ["NHMoEError", "Config", "Layout", "config_from", "load", "validate", "workspace_size",
           "workspace_layout", "shared_workspace_size", "route", "route_noalloc", "route_permute", "permute", "forward", "experts_up", "experts_down", "shared", "forward_nvfp4", "shared_nvfp4", "nvfp4_weight",
           "zero_acc", "finalize", "latent_config", "latent_workspace_size",
           "latent_in", "latent_out", "reset_status", "check_device", "selftest_timeout", "library_path", "NemotronHMoE"]

NH_OK, NH_ERR_INVALID_ARG, NH_ERR_UNSUPPORTED, NH_ERR_CUDA, NH_ERR_TIMEOUT, NH_ERR_DEVICE_CHECK = range(6)
STATUS_NAMES = {0: "NH_OK", 1: "NH_ERR_INVALID_ARG", 2: "NH_ERR_UNSUPPORTED", 3: "NH_ERR_CUDA",
                4: "NH_ERR_TIMEOUT", 5: "NH_ERR_DEVICE_CHECK"}
NH_F32, NH_BF16 = 0, 1


class NHMoEError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class Config(ctypes.Structure):
    """nh_moe_config (field names of the model's config.json)."""
    _fields_ = [("hidden_size", ctypes.c_int32), ("n_routed_experts", ctypes.c_int32),
                ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32),
                ("num_experts_per_tok", ctypes.c_int32), ("moe_intermediate_size", ctypes.c_int32),
                ("moe_shared_expert_intermediate_size", ctypes.c_int32),
                ("n_shared_experts", ctypes.c_int32), ("norm_topk_prob", ctypes.c_int32),
                ("routed_scaling_factor", ctypes.c_float), ("dtype", ctypes.c_int32),
                ("group_score", ctypes.c_int32), ("weight_format", ctypes.c_int32),
                ("latent_size", ctypes.c_int32)]


class NvFp4Weight(ctypes.Structure):
    """nh_nvfp4_weight: device pointers of one stacked NVFP4 tensor."""
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("global_scale", ctypes.c_void_p)]


NH_WEIGHTS_NATIVE, NH_WEIGHTS_NVFP4 = 0, 1


class Layout(ctypes.Structure):
    """nh_moe_ws_layout: byte offsets of the routed-path workspace regions."""
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "total_bytes", "status", "logits", "router_w", "counts", "offsets", "chunk_counts", "perm_token",
        "perm_w", "inv_row", "tiles", "num_tiles", "x_perm", "h", "ready")] + [
        ("rows_alloc", ctypes.c_int64), ("tile_rows", ctypes.c_int32),
        ("max_tiles", ctypes.c_int32), ("n_chunks", ctypes.c_int32), ("swap_ab", ctypes.c_int32),
        ("x_direct", ctypes.c_int32)]


def config_from(c, group_score: int = 0) -> Config:
    """Build the C struct from any object with the config.json attribute names
    (and ``dtype`` in {"bf16", "f32"})."""
    if isinstance(c, Config):
        return c
    dt = getattr(c, "dtype", "bf16")
    return Config(int(c.hidden_size), int(c.n_routed_experts), int(c.n_group), int(c.topk_group),
                  int(c.num_experts_per_tok), int(c.moe_intermediate_size),
                  int(c.moe_shared_expert_intermediate_size), int(c.n_shared_experts),
                  int(bool(c.norm_topk_prob)), float(c.routed_scaling_factor),
                  NH_BF16 if dt in ("bf16", NH_BF16) else NH_F32,
                  int(getattr(c, "group_score", group_score)),
                  NH_WEIGHTS_NVFP4 if getattr(c, "weight_format", "native") in ("nvfp4", 1)
                  else NH_WEIGHTS_NATIVE, int(getattr(c, "latent_size", 0) or 0))


_lock = threading.Lock()
_lib = None

_EXPORTS = ["nh_moe_validate", "nh_moe_workspace_size", "nh_moe_workspace_layout",
            "nh_moe_shared_workspace_size", "nh_moe_route", "nh_moe_route_noalloc", "nh_moe_route_permute",
            "nh_moe_permute", "nh_moe_forward", "nh_moe_experts_up", "nh_moe_experts_down",
            "nh_moe_forward_nvfp4", "nh_moe_shared", "nh_moe_shared_store", "nh_moe_shared_nvfp4",
            "nh_moe_zero_acc",
            "nh_moe_finalize",
            "nh_moe_latent_config", "nh_moe_latent_workspace_size", "nh_moe_latent_in",
            "nh_moe_latent_out", "nh_moe_reset_status", "nh_moe_check_device",
            "nh_moe_selftest_timeout",
            "nh_last_error", "nh_version"]


def library_path() -> str:
    return _build.LIB


def load():
    """Build (if sources changed) and load libnhmoe.so; raise if impossible."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = _build.build()
        lib = ctypes.CDLL(path)
        P, S, I64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64
        C = ctypes.POINTER(Config)
        sig = {
            "nh_moe_validate": [C],
            "nh_moe_workspace_size": [C, I64, ctypes.POINTER(S)],
            "nh_moe_workspace_layout": [C, I64, ctypes.POINTER(Layout)],
            "nh_moe_shared_workspace_size": [C, I64, ctypes.POINTER(S)],
            "nh_moe_route": [C, I64, P, P, P, P, P, P, S, P],
            "nh_moe_route_noalloc": [C, I64, P, P, P, P, P, P],
            "nh_moe_route_permute": [C, I64, P, P, P, P, P, P, S, P],
            "nh_moe_permute": [C, I64, P, P, P, P, S, P],
            "nh_moe_forward": [C, I64, P, P, P, P, S, P, P],
            "nh_moe_experts_up": [C, I64, P, P, P, S, P],
            "nh_moe_experts_down": [C, I64, P, P, S, P, P],
            "nh_moe_shared": [C, I64, P, P, P, P, P, S, P],
            "nh_moe_forward_nvfp4": [C, I64, P, ctypes.POINTER(NvFp4Weight),
                                     ctypes.POINTER(NvFp4Weight), P, S, P, P],
            "nh_moe_shared_nvfp4": [C, I64, P, ctypes.POINTER(NvFp4Weight),
                                    ctypes.POINTER(NvFp4Weight), P, P, S, P],
            "nh_moe_zero_acc": [C, I64, P, P],
            "nh_moe_finalize": [C, I64, P, P, P],
            "nh_moe_latent_config": [C, C],
            "nh_moe_latent_workspace_size": [C, I64, ctypes.POINTER(S)],
            "nh_moe_latent_in": [C, I64, P, P, P, P, S, P],
            "nh_moe_latent_out": [C, I64, P, P, P, P, S, P],
            "nh_moe_check_device": [P, P],
            "nh_moe_reset_status": [P, P],
            "nh_moe_selftest_timeout": [P, ctypes.c_uint64, P],
        }
        for name, args in sig.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        lib.nh_last_error.restype = ctypes.c_char_p
        lib.nh_version.restype = ctypes.c_char_p
        _lib = lib
        return lib


def _check(rc: int):
    if rc != NH_OK:
        raise NHMoEError(rc, load().nh_last_error().decode())


def _p(t):
    """Device pointer of a tensor (or None)."""
    if t is None:
        return None
    if hasattr(t, "data_ptr"):
        if not t.is_contiguous():
            raise ValueError("tensors passed to libnhmoe must be contiguous")
        return ctypes.c_void_p(t.data_ptr())
    return ctypes.c_void_p(int(t))


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if hasattr(stream, "cuda_stream"):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _nbytes(t):
    return t.numel() * t.element_size()


def validate(cfg):
    _check(load().nh_moe_validate(ctypes.byref(config_from(cfg))))


def workspace_size(cfg, T: int) -> int:
    n = ctypes.c_size_t()
    _check(load().nh_moe_workspace_size(ctypes.byref(config_from(cfg)), T, ctypes.byref(n)))
    return n.value


def workspace_layout(cfg, T: int) -> Layout:
    lay = Layout()
    _check(load().nh_moe_workspace_layout(ctypes.byref(config_from(cfg)), T, ctypes.byref(lay)))
    return lay


def shared_workspace_size(cfg, T: int) -> int:
    n = ctypes.c_size_t()
    _check(load().nh_moe_shared_workspace_size(ctypes.byref(config_from(cfg)), T,
                                               ctypes.byref(n)))
    return n.value


def route(cfg, x, w_router, bias, topk_idx, topk_w, ws, stream=None):
    c = config_from(cfg)
    _check(load().nh_moe_route(ctypes.byref(c), x.shape[0], _p(x), _p(w_router), _p(bias),
                               _p(topk_idx), _p(topk_w), _p(ws), _nbytes(ws), _stream(stream)))


def route_noalloc(cfg, x, w_router, bias, topk_idx, topk_w, stream=None):
    """Router of decode-sized batches (T <= 32) without a workspace argument: its
    scratch is a fixed array inside the library (see nh_moe_route_noalloc)."""
    c = config_from(cfg)
    _check(load().nh_moe_route_noalloc(ctypes.byref(c), x.shape[0], _p(x), _p(w_router),
                                       _p(bias), _p(topk_idx), _p(topk_w), _stream(stream)))


def route_permute(cfg, x, w_router, bias, topk_idx, topk_w, ws, stream=None):
    """route + permute in one call (one kernel for T <= 32)."""
    c = config_from(cfg)
    _check(load().nh_moe_route_permute(ctypes.byref(c), x.shape[0], _p(x), _p(w_router), _p(bias),
                                       _p(topk_idx), _p(topk_w), _p(ws), _nbytes(ws),
                                       _stream(stream)))


def permute(cfg, x, topk_idx, topk_w, ws, stream=None):
    c = config_from(cfg)
    _check(load().nh_moe_permute(ctypes.byref(c), x.shape[0], _p(x), _p(topk_idx), _p(topk_w),
                                 _p(ws), _nbytes(ws), _stream(stream)))


def forward(cfg, x, w_up, w_down, ws, y_acc, stream=None):
    """Routed experts: y_acc[token] += the token's weighted expert outputs (float32)."""
    c = config_from(cfg)
    _check(load().nh_moe_forward(ctypes.byref(c), x.shape[0], _p(x), _p(w_up), _p(w_down), _p(ws),
                                 _nbytes(ws), _p(y_acc), _stream(stream)))


def experts_up(cfg, x, w_up, ws, stream=None):
    c = config_from(cfg)
    _check(load().nh_moe_experts_up(ctypes.byref(c), x.shape[0], _p(x), _p(w_up), _p(ws),
                                    _nbytes(ws), _stream(stream)))


def experts_down(cfg, T: int, w_down, ws, y_acc, stream=None):
    c = config_from(cfg)
    _check(load().nh_moe_experts_down(ctypes.byref(c), T, _p(w_down), _p(ws), _nbytes(ws),
                                      _p(y_acc), _stream(stream)))


def shared(cfg, x, w_shared_up, w_shared_down, y_acc, ws_shared, stream=None):
    """Shared expert: y_acc += relu(x W_su^T)^2 W_sd^T (float32)."""
    c = config_from(cfg)
    _check(load().nh_moe_shared(ctypes.byref(c), x.shape[0], _p(x), _p(w_shared_up),
                                _p(w_shared_down), _p(y_acc), _p(ws_shared),
                                _nbytes(ws_shared), _stream(stream)))


def shared_store(cfg, x, w_shared_up, w_shared_down, y_acc, ws_shared, stream=None):
    """Shared expert as y_acc's starting value: y_acc = relu(x W_su^T)^2 W_sd^T."""
    c = config_from(cfg)
    _check(load().nh_moe_shared_store(ctypes.byref(c), x.shape[0], _p(x), _p(w_shared_up),
                                      _p(w_shared_down), _p(y_acc), _p(ws_shared),
                                      _nbytes(ws_shared), _stream(stream)))


def nvfp4_weight(codes, scales, global_scale) -> NvFp4Weight:
    """Struct of device pointers for one stacked NVFP4 tensor (tensors stay owned by the caller)."""
    return NvFp4Weight(codes.data_ptr(), scales.data_ptr(), global_scale.data_ptr())


def forward_nvfp4(cfg, x, w_up, w_down, ws, y_acc, stream=None):
    """nh_moe_forward with NVFP4 weights; w_up / w_down are NvFp4Weight structs."""
    c = config_from(cfg)
    _check(load().nh_moe_forward_nvfp4(ctypes.byref(c), x.shape[0], _p(x), ctypes.byref(w_up),
                                       ctypes.byref(w_down), _p(ws), _nbytes(ws), _p(y_acc),
                                       _stream(stream)))


def shared_nvfp4(cfg, x, w_shared_up, w_shared_down, y_acc, ws_shared, stream=None):
    c = config_from(cfg)
    _check(load().nh_moe_shared_nvfp4(ctypes.byref(c), x.shape[0], _p(x), ctypes.byref(w_shared_up),
                                      ctypes.byref(w_shared_down), _p(y_acc), _p(ws_shared),
                                      _nbytes(ws_shared), _stream(stream)))


def zero_acc(cfg, T: int, y_acc, stream=None):
    """y_acc = 0 ([T, hidden_size] float32), asynchronously on `stream`."""
    c = config_from(cfg)
    _check(load().nh_moe_zero_acc(ctypes.byref(c), T, _p(y_acc), _stream(stream)))


def finalize(cfg, T: int, y_acc, y, stream=None):
    """y = dtype(y_acc): the one rounding of the block output."""
    c = config_from(cfg)
    _check(load().nh_moe_finalize(ctypes.byref(c), T, _p(y_acc), _p(y), _stream(stream)))


def latent_config(cfg) -> Config:
    """The expert-width config the routed-expert calls of a latent block take
    (hidden_size = latent_size, no latent projections, no shared expert)."""
    c = config_from(cfg)
    out = Config()
    _check(load().nh_moe_latent_config(ctypes.byref(c), ctypes.byref(out)))
    return out


def latent_workspace_size(cfg, T: int) -> int:
    c = config_from(cfg)
    n = ctypes.c_size_t()
    _check(load().nh_moe_latent_workspace_size(ctypes.byref(c), T, ctypes.byref(n)))
    return n.value


def latent_in(cfg, x, w_latent_fc1, x_lat, ws_latent, stream=None):
    """x_lat = dtype(x W_fc1^T)."""
    c = config_from(cfg)
    _check(load().nh_moe_latent_in(ctypes.byref(c), x.shape[0], _p(x), _p(w_latent_fc1),
                                   _p(x_lat), _p(ws_latent), _nbytes(ws_latent), _stream(stream)))


def latent_out(cfg, T: int, y_lat, w_latent_fc2, y_acc, ws_latent, stream=None):
    """y_acc += y_lat W_fc2^T (y_acc = ... without a shared expert), float32."""
    c = config_from(cfg)
    _check(load().nh_moe_latent_out(ctypes.byref(c), T, _p(y_lat), _p(w_latent_fc2), _p(y_acc),
                                    _p(ws_latent), _nbytes(ws_latent), _stream(stream)))


def reset_status(ws, stream=None):
    """Clear a workspace's status word (asynchronously, on `stream`)."""
    _check(load().nh_moe_reset_status(_p(ws), _stream(stream)))


def check_device(ws, stream=None) -> int:
    """Synchronise the stream and return the workspace status word (raises on CUDA errors)."""
    rc = load().nh_moe_check_device(_p(ws), _stream(stream))
    if rc == NH_ERR_CUDA:
        _check(rc)
    return rc


def selftest_timeout(ws, timeout_ns: int, stream=None):
    _check(load().nh_moe_selftest_timeout(_p(ws), int(timeout_ns), _stream(stream)))


def last_error() -> str:
    return load().nh_last_error().decode()


from .block import NemotronHMoE  # noqa: E402
