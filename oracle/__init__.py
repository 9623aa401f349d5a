"""CPU oracle of the Nemotron-H non-gated MoE block forward (fp64).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference legs may import this package.  It shares
no code with ``non_gated_relu_b200`` and never imports it.

The arithmetic lives in ``nh_oracle.c`` (plain single-threaded loops in
double precision; see its header for the passages each step follows).  This
module builds that file with gcc and marshals numpy arrays into it.  One
more step, the token permute, is the plain stable counting sort written out
below in numpy.

Every function here is pinned by ``-m "not gpu"`` tests against values that
do not come from the oracle itself: a hand-worked routing example, brute
force over every group / expert subset, closed-form special cases, a dense
masked formulation of the combine, and invariants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nh_oracle.c")
_LIB = os.path.join(_HERE, "libnh_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc -O2 (no fast-math, no OpenMP, no intrinsics)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int64), ("E", ctypes.c_int64), ("G", ctypes.c_int64),
                ("tg", ctypes.c_int64), ("k", ctypes.c_int64), ("I", ctypes.c_int64),
                ("S", ctypes.c_int64), ("n_shared", ctypes.c_int64), ("norm", ctypes.c_int64),
                ("alpha", ctypes.c_double), ("dtype", ctypes.c_int64),
                ("group_score", ctypes.c_int64)]


class _Wt(ctypes.Structure):
    """nho_wt: one stacked weight tensor [n_mat][rows][cols] (float32, bf16 or NVFP4)."""
    _fields_ = [("format", ctypes.c_int64), ("data", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("global_", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("scale_pitch", ctypes.c_int64)]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            lib.nho_check_config.argtypes = [ctypes.POINTER(_Cfg)]
            lib.nho_route.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int64, P, P, P, P, P, P, P]
            lib.nho_forward.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int64, P, P, P, P, P, P,
                                        P, P, P, P, ctypes.c_int64, P, P, P]
            W = ctypes.POINTER(_Wt)
            lib.nho_forward_wt.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int64, P, P, P, W, W, W,
                                           W, P, P, P, ctypes.c_int64, P, P, P]
            lib.nho_dequant.argtypes = [W, ctypes.c_int64, P]
            lib.nho_forward_latent.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int64,
                                               ctypes.c_int64, P, P, P, W, W, W, W, P, P, P, P,
                                               P, ctypes.c_int64, P, P, P]
            _lib = lib
    return _lib


def _swap_library(path):
    """Load the oracle from another build of its source (used by the mutation
    tests, which compile deliberately broken copies); returns the previous
    handle so the caller can restore it with ``_restore_library``."""
    global _lib
    prev = _load()
    lib = ctypes.CDLL(path)
    for name in ("nho_check_config", "nho_route", "nho_forward", "nho_forward_wt", "nho_dequant"):
        getattr(lib, name).argtypes = getattr(prev, name).argtypes
    with _lock:
        _lib = lib
    return prev


def _restore_library(prev):
    global _lib
    with _lock:
        _lib = prev


def _cfg(cfg, group_score: int = 0) -> _Cfg:
    return _Cfg(cfg.H, cfg.E, cfg.G, cfg.tg, cfg.k, cfg.I, cfg.S, int(cfg.n_shared_experts),
                int(bool(cfg.norm_topk_prob)), float(cfg.routed_scaling_factor),
                1 if cfg.dtype == "bf16" else 0, int(group_score))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _stored(a, dtype):
    want = np.uint16 if dtype == "bf16" else np.float32
    a = np.ascontiguousarray(a)
    if a.dtype != want:
        raise TypeError(f"expected {want} storage, got {a.dtype}")
    return a


class OracleError(RuntimeError):
    pass


def check_config(cfg, group_score: int = 0) -> int:
    return _load().nho_check_config(ctypes.byref(_cfg(cfg, group_score)))


def route(cfg, x, w_router, bias=None, group_score: int = 0):
    """Grouped top-k sigmoid routing of every token.

    Returns (topk_idx int32 [T,k], topk_w float64 [T,k], gap_group [T], gap_expert [T]).
    """
    lib = _load()
    c = _cfg(cfg, group_score)
    x = _stored(x, cfg.dtype)
    wr = np.ascontiguousarray(w_router, np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    T = x.shape[0]
    idx = np.zeros((T, cfg.k), np.int32)
    w = np.zeros((T, cfg.k), np.float64)
    gg = np.zeros(T, np.float64)
    ge = np.zeros(T, np.float64)
    rc = lib.nho_route(ctypes.byref(c), T, _ptr(x), _ptr(wr), _ptr(b), _ptr(idx), _ptr(w),
                       _ptr(gg), _ptr(ge))
    if rc:
        raise OracleError(f"nho_route failed ({rc})")
    return idx, w, gg, ge


def route_parallel(cfg, x, w_router, bias=None, threads: int = 8, group_score: int = 0):
    """``route`` over token shards in threads (each shard is the single-threaded oracle)."""
    T = x.shape[0]
    if T < 64 or threads <= 1:
        return route(cfg, x, w_router, bias, group_score)
    bounds = np.linspace(0, T, threads + 1).astype(int)
    with ThreadPoolExecutor(threads) as ex:
        parts = list(ex.map(lambda i: route(cfg, x[bounds[i]:bounds[i + 1]], w_router, bias,
                                            group_score), range(threads)))
    return tuple(np.concatenate([p[i] for p in parts]) for i in range(4))


def _wt_nvfp4(q, rows, cols):
    codes, scales, g = (np.ascontiguousarray(q[0], np.uint8), np.ascontiguousarray(q[1], np.uint8),
                        np.ascontiguousarray(q[2], np.float32))
    keep = (codes, scales, g)
    return _Wt(2, codes.ctypes.data, scales.ctypes.data, g.ctypes.data, rows, cols,
               scales.shape[-1]), keep


def dequant_nvfp4(q, rows, cols, mat=0):
    """Dense float64 [rows, cols] of matrix `mat` of an NVFP4 tensor (codes, scales, global)."""
    w, keep = _wt_nvfp4(q, rows, cols)
    out = np.zeros((rows, cols), np.float64)
    rc = _load().nho_dequant(ctypes.byref(w), mat, _ptr(out))
    if rc:
        raise OracleError(f"nho_dequant failed ({rc})")
    return out


def _forward_nvfp4(inp, tok, oi, ow, group_score):
    cfg = inp.cfg
    lib = _load()
    c = _cfg(cfg, group_score)
    n = tok.shape[0]
    y = np.zeros((n, cfg.H), np.float64)
    idx = np.zeros((n, cfg.k), np.int32)
    w = np.zeros((n, cfg.k), np.float64)
    q = inp.nvfp4
    up, k1 = _wt_nvfp4(q["up"], cfg.I, cfg.H)
    dn, k2 = _wt_nvfp4(q["down"], cfg.H, cfg.I)
    su = sd = None
    keep = [k1, k2]
    if cfg.n_shared_experts:
        su, k3 = _wt_nvfp4(q["shared_up"], cfg.S, cfg.H)
        sd, k4 = _wt_nvfp4(q["shared_down"], cfg.H, cfg.S)
        keep += [k3, k4]
    x = _stored(inp.x, cfg.dtype)
    wr = np.ascontiguousarray(inp.w_router, np.float32)
    b = None if inp.bias is None else np.ascontiguousarray(inp.bias, np.float32)
    rc = lib.nho_forward_wt(ctypes.byref(c), inp.x.shape[0], _ptr(x), _ptr(wr), _ptr(b),
                            ctypes.byref(up), ctypes.byref(dn),
                            ctypes.byref(su) if su is not None else None,
                            ctypes.byref(sd) if sd is not None else None,
                            _ptr(oi), _ptr(ow), _ptr(tok), n, _ptr(y), _ptr(idx), _ptr(w))
    if rc:
        raise OracleError(f"nho_forward_wt failed ({rc})")
    return y, idx, w


def _wt_native(a, dtype, rows, cols):
    a = _stored(a, dtype)
    return _Wt(1 if dtype == "bf16" else 0, a.ctypes.data, None, None, rows, cols, 0), a


def _forward_latent(inp, tok, oi, ow, group_score):
    """Latent block (nho_forward_latent): routed experts between
    fc1_latent_proj and fc2_latent_proj; parity of this reading is unpinned."""
    cfg = inp.cfg
    lib = _load()
    c = _cfg(cfg, group_score)
    n = tok.shape[0]
    L = cfg.latent_size
    y = np.zeros((n, cfg.H), np.float64)
    idx = np.zeros((n, cfg.k), np.int32)
    w = np.zeros((n, cfg.k), np.float64)
    keep = []
    if getattr(inp, "nvfp4", None) is not None:
        q = inp.nvfp4
        up, k1 = _wt_nvfp4(q["up"], cfg.I, L)
        dn, k2 = _wt_nvfp4(q["down"], L, cfg.I)
        su = sd = None
        keep += [k1, k2]
        if cfg.n_shared_experts:
            su, k3 = _wt_nvfp4(q["shared_up"], cfg.S, cfg.H)
            sd, k4 = _wt_nvfp4(q["shared_down"], cfg.H, cfg.S)
            keep += [k3, k4]
    else:
        up, k1 = _wt_native(inp.w_up, cfg.dtype, cfg.I, L)
        dn, k2 = _wt_native(inp.w_down, cfg.dtype, L, cfg.I)
        su = sd = None
        keep += [k1, k2]
        if cfg.n_shared_experts:
            su, k3 = _wt_native(inp.w_shared_up, cfg.dtype, cfg.S, cfg.H)
            sd, k4 = _wt_native(inp.w_shared_down, cfg.dtype, cfg.H, cfg.S)
            keep += [k3, k4]
    x = _stored(inp.x, cfg.dtype)
    wl1 = _stored(inp.w_latent_fc1, cfg.dtype)
    wl2 = _stored(inp.w_latent_fc2, cfg.dtype)
    wr = np.ascontiguousarray(inp.w_router, np.float32)
    b = None if inp.bias is None else np.ascontiguousarray(inp.bias, np.float32)
    rc = lib.nho_forward_latent(ctypes.byref(c), L, inp.x.shape[0], _ptr(x), _ptr(wr), _ptr(b),
                                ctypes.byref(up), ctypes.byref(dn),
                                ctypes.byref(su) if su is not None else None,
                                ctypes.byref(sd) if sd is not None else None,
                                _ptr(wl1), _ptr(wl2), _ptr(oi), _ptr(ow), _ptr(tok), n, _ptr(y),
                                _ptr(idx), _ptr(w))
    if rc:
        raise OracleError(f"nho_forward_latent failed ({rc})")
    return y, idx, w


def forward(inp, tokens=None, override_idx=None, override_w=None, group_score: int = 0):
    """Block output y (float64 [n_tok, H]) for the listed tokens (default: all).

    ``inp`` is a ``synth.MoEInputs``.  With ``override_idx``/``override_w``
    ([n_tok, k]) the routing is taken from the caller instead of computed.
    Returns (y, idx_used, w_used).
    """
    cfg = inp.cfg
    lib = _load()
    c = _cfg(cfg, group_score)
    T = inp.x.shape[0]
    tok = np.arange(T, dtype=np.int64) if tokens is None else np.ascontiguousarray(tokens, np.int64)
    n = tok.shape[0]
    y = np.zeros((n, cfg.H), np.float64)
    idx = np.zeros((n, cfg.k), np.int32)
    w = np.zeros((n, cfg.k), np.float64)
    oi = ow = None
    if override_idx is not None:
        oi = np.ascontiguousarray(override_idx, np.int32).reshape(n, cfg.k)
        ow = np.ascontiguousarray(override_w, np.float64).reshape(n, cfg.k)
    if getattr(cfg, "latent_size", 0):
        return _forward_latent(inp, tok, oi, ow, group_score)
    if getattr(inp, "nvfp4", None) is not None:
        return _forward_nvfp4(inp, tok, oi, ow, group_score)
    x = _stored(inp.x, cfg.dtype)
    args = [_stored(a, cfg.dtype) if a is not None else None
            for a in (inp.w_up, inp.w_down, inp.w_shared_up, inp.w_shared_down)]
    wr = np.ascontiguousarray(inp.w_router, np.float32)
    b = None if inp.bias is None else np.ascontiguousarray(inp.bias, np.float32)
    rc = lib.nho_forward(ctypes.byref(c), T, _ptr(x), _ptr(wr), _ptr(b), *[_ptr(a) for a in args],
                         _ptr(oi), _ptr(ow), _ptr(tok), n, _ptr(y), _ptr(idx), _ptr(w))
    if rc:
        raise OracleError(f"nho_forward failed ({rc})")
    return y, idx, w


def forward_parallel(inp, tokens=None, override_idx=None, override_w=None, threads: int = 8,
                     group_score: int = 0):
    """``forward`` over token shards in threads (ctypes releases the GIL)."""
    T = inp.x.shape[0]
    tok = np.arange(T, dtype=np.int64) if tokens is None else np.asarray(tokens, np.int64)
    n = tok.shape[0]
    if n < 2 or threads <= 1:
        return forward(inp, tok, override_idx, override_w, group_score)
    nt = min(threads, n)
    bounds = np.linspace(0, n, nt + 1).astype(int)

    def one(i):
        s = slice(bounds[i], bounds[i + 1])
        oi = None if override_idx is None else np.asarray(override_idx)[s]
        ow = None if override_w is None else np.asarray(override_w)[s]
        return forward(inp, tok[s], oi, ow, group_score)

    with ThreadPoolExecutor(nt) as ex:
        parts = list(ex.map(one, range(nt)))
    return tuple(np.concatenate([p[i] for p in parts]) for i in range(3))


def permute(topk_idx, topk_w, E: int):
    """Token permute: stable counting sort of the (token, slot) assignments by expert.

    The routed experts are applied expert by expert (MLX ``SwitchMLP`` with
    ``fc1``/``fc2`` indexed by the router's expert ids, exo commit "Add
    support for Nemotron sharding"); the assignments are grouped per expert
    in (token, slot) order.  Returns dict with
      counts [E], offsets [E+1], perm_token [T*k], perm_slot [T*k],
      perm_w [T*k], inv_row [T, k] (row of assignment (t, j)).
    """
    idx = np.asarray(topk_idx)
    T, k = idx.shape
    flat = idx.reshape(-1).astype(np.int64)
    counts = np.zeros(E, np.int64)
    for e in flat:                       # histogram
        counts[e] += 1
    offsets = np.zeros(E + 1, np.int64)  # exclusive scan
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    fill = offsets[:-1].copy()
    perm = np.zeros(T * k, np.int64)
    inv = np.zeros(T * k, np.int64)
    for a, e in enumerate(flat):         # stable scatter in (t, j) order
        perm[fill[e]] = a
        inv[a] = fill[e]
        fill[e] += 1
    wflat = np.asarray(topk_w).reshape(-1)
    return {"counts": counts, "offsets": offsets, "perm_token": perm // k, "perm_slot": perm % k,
            "perm_w": wflat[perm], "inv_row": inv.reshape(T, k)}
