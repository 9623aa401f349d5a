"""Block-level API: ``NemotronHMoE(cfg, weights...)(x) -> y``.

The Nemotron-H MoE block (``NemotronHMoE.__call__(x) -> y`` with a
``switch_mlp`` of routed experts and a ``shared_experts`` NemotronHMLP, exo
commit "Add support for Nemotron sharding", nemotron_h.pyi) on one GPU.  One
call runs, on the caller's stream and a side stream:

    side: y_acc = 0 --+-> shared expert: y_acc += shared(x) ----------+
    main: route + permute -> forward: y_acc += routed experts (x) ---+-> finalize: y = dtype(y_acc)
                      (forward waits for y_acc = 0)

The shared expert runs beside the routed path at every size: at decode its
GEMVs stream their weights while the router runs, and at prefill its GEMMs take
the SMs that the routing and permute kernels leave idle (measured faster than
running it in turn on one stream, from 6144 to 16384 tokens).  For bf16 decode
batches (at most 32 tokens) the router is launched before the shared expert, so
that its blocks reach the SMs first; the streams and their joins are the same.
For more than
32 tokens with native weights its down projection writes y_acc's starting
value instead of adding into zeros (no fill, no read of the zeros), and the
routed down projection waits for it:

    side: shared expert: y_acc = shared(x) ----------------------------+
    main: route + permute -> experts_up -> (wait) experts_down: y_acc += routed -> finalize

With latent projections (config ``latent_size`` L > 0; the modules
fc1_latent_proj / fc2_latent_proj of the ModelOpt descriptor
NemotronHMoELayerDescriptor) the routed experts run in width L:

    side: y_acc = 0, y_lat_acc = 0 -> shared expert(x) into y_acc ------+
    main: route(x) -> fc1: x_lat -> permute + forward into y_lat_acc      |
          -> y_lat = dtype(y_lat_acc) --+-> fc2: y_acc += y_lat W_fc2^T -> y = dtype(y_acc)

All arithmetic happens in libnhmoe's kernels; this class only owns buffers,
streams, events and (optionally) a CUDA graph of the call sequence.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, Optional

import numpy as np
import torch

from . import (check_device, config_from, experts_down, experts_up, finalize, forward,
               forward_nvfp4, latent_config,
               latent_in, latent_out, latent_workspace_size, nvfp4_weight, permute, reset_status,
               route, route_permute, shared, shared_nvfp4, shared_store, shared_workspace_size,
               validate,
               workspace_layout, workspace_size, zero_acc, NH_BF16, NH_WEIGHTS_NVFP4)


def _to_device(a, dtype: torch.dtype, device) -> torch.Tensor:
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if a.dtype == np.uint16:
            t = t.view(torch.bfloat16)
    else:
        t = a
    if t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    return t.to(device).contiguous()


@dataclass
class Buffers:
    T: int
    ws: torch.Tensor
    ws_shared: Optional[torch.Tensor]
    topk_idx: torch.Tensor
    topk_w: torch.Tensor
    y_acc: torch.Tensor                      # float32 [T, H]: shared + weighted routed experts
    y: torch.Tensor
    # latent blocks: routing workspace (full width), projection workspace,
    # x_lat / y_lat [T, L] and the float32 accumulator of the routed experts [T, L]
    ws_route: Optional[torch.Tensor] = None
    ws_lat: Optional[torch.Tensor] = None
    x_lat: Optional[torch.Tensor] = None
    y_lat: Optional[torch.Tensor] = None
    y_lat_acc: Optional[torch.Tensor] = None


class NemotronHMoE:
    """One MoE block with resident weights.

    Weights use the PyTorch Linear layout: ``w_router [E, H]`` float32,
    ``w_up [E, I, H]``, ``w_down [E, H, I]``, ``w_shared_up [S, H]``,
    ``w_shared_down [H, S]`` in the block dtype (bf16 or float32), and an
    optional router correction bias ``[E]`` float32.  numpy uint16 arrays are
    taken as bf16 bit patterns.

    libnhmoe launches on the current CUDA device, so call the block with its
    own device current (``torch.cuda.set_device`` or a ``torch.cuda.device``
    context), as one process per GPU does.
    """

    def __init__(self, cfg, w_router, w_up=None, w_down=None, w_shared_up=None,
                 w_shared_down=None, bias=None, device=None, nvfp4=None, w_latent_fc1=None,
                 w_latent_fc2=None):
        self.cfg = cfg
        self.c = config_from(cfg)
        validate(self.c)
        self.device = torch.device(device if device is not None else "cuda")
        if self.device.type != "cuda":
            raise ValueError("NemotronHMoE runs on a CUDA device only")
        self.dtype = torch.bfloat16 if self.c.dtype == NH_BF16 else torch.float32
        self.H = self.c.hidden_size
        self.k = self.c.num_experts_per_tok
        self.has_shared = bool(self.c.n_shared_experts)
        self.w_router = _to_device(w_router, torch.float32, self.device)
        self.bias = _to_device(bias, torch.float32, self.device)
        self.nvfp4 = self.c.weight_format == NH_WEIGHTS_NVFP4
        if self.nvfp4:
            # {"up", "down", "shared_up", "shared_down"} -> (codes, scales, global)
            if nvfp4 is None:
                raise ValueError("config has NVFP4 weights: pass nvfp4={...}")
            self._q4_tensors = {}
            self.q4 = {}
            for name, (codes, scales, glob) in nvfp4.items():
                t = tuple(torch.as_tensor(a).to(self.device).contiguous()
                          for a in (codes, scales, glob))
                self._q4_tensors[name] = t
                self.q4[name] = nvfp4_weight(*t)
            self.w_up = self.w_down = self.w_shared_up = self.w_shared_down = None
            if self.has_shared and ("shared_up" not in self.q4 or "shared_down" not in self.q4):
                raise ValueError("config has a shared expert but no shared weights were given")
        else:
            self.w_up = _to_device(w_up, self.dtype, self.device)
            self.w_down = _to_device(w_down, self.dtype, self.device)
            self.w_shared_up = _to_device(w_shared_up, self.dtype, self.device)
            self.w_shared_down = _to_device(w_shared_down, self.dtype, self.device)
            if self.has_shared and (self.w_shared_up is None or self.w_shared_down is None):
                raise ValueError("config has a shared expert but no shared weights were given")
        self.latent = bool(self.c.latent_size)
        if self.latent:
            # routed-expert calls take the expert-width config
            self.c_exp = latent_config(self.c)
            self.L = self.c.latent_size
            self.w_latent_fc1 = _to_device(w_latent_fc1, self.dtype, self.device)
            self.w_latent_fc2 = _to_device(w_latent_fc2, self.dtype, self.device)
            if self.w_latent_fc1 is None or self.w_latent_fc2 is None:
                raise ValueError("config has latent_size > 0: pass w_latent_fc1 / w_latent_fc2")
        else:
            self.c_exp = self.c
        with torch.cuda.device(self.device):
            # the routed path (router -> experts -> finalize) is the critical
            # path: its kernels run on the highest-priority stream, so pending
            # CTAs start before those of the shared expert on `side`
            self.hi = torch.cuda.Stream(priority=-5)
            self.side = torch.cuda.Stream()
        self._bufs: Dict[int, Buffers] = {}
        self._graphs: Dict[int, tuple] = {}
        self._host: Dict[int, tuple] = {}

    # ------------------------------------------------------------------ buffers
    def buffers(self, T: int, slot: int = 0) -> Buffers:
        """Device buffers of a call with T tokens (``slot`` > 0: a further set, for
        calls in flight together, see ``pipeline``)."""
        b = self._bufs.get((T, slot))
        if b is None:
            dev = self.device
            ws = torch.empty(workspace_size(self.c_exp, T), dtype=torch.uint8, device=dev)
            wss = None
            if self.has_shared:
                wss = torch.empty(shared_workspace_size(self.c, T), dtype=torch.uint8, device=dev)
            b = Buffers(T, ws, wss,
                        torch.empty((T, self.k), dtype=torch.int32, device=dev),
                        torch.empty((T, self.k), dtype=torch.float32, device=dev),
                        torch.empty((T, self.H), dtype=torch.float32, device=dev),
                        torch.empty((T, self.H), dtype=self.dtype, device=dev))
            if self.latent:
                b.ws_route = torch.empty(max(256, workspace_layout(self.c, T).counts),
                                         dtype=torch.uint8, device=dev)
                b.ws_lat = torch.empty(latent_workspace_size(self.c, T), dtype=torch.uint8,
                                       device=dev)
                b.x_lat = torch.empty((T, self.L), dtype=self.dtype, device=dev)
                b.y_lat = torch.empty((T, self.L), dtype=self.dtype, device=dev)
                b.y_lat_acc = torch.empty((T, self.L), dtype=torch.float32, device=dev)
            self._bufs[(T, slot)] = b
        return b

    # ------------------------------------------------------------------ compute
    def forward(self, x: torch.Tensor, bufs: Optional[Buffers] = None,
                nvtx: bool = False, partial: bool = False) -> torch.Tensor:
        """y for a device tensor x [T, H]; returns the buffer-owned y [T, H].
        ``nvtx`` wraps each call in an NVTX range of its name (for profilers).
        ``partial`` (a tensor-parallel shard) returns instead the float32
        accumulator y_acc of this shard's contributions, unrounded, for an
        all-reduce."""
        T = x.shape[0]
        b = bufs or self.buffers(T)
        caller = torch.cuda.current_stream(self.device)
        main = self.hi
        push = torch.cuda.nvtx.range_push if nvtx else (lambda name: None)
        pop = torch.cuda.nvtx.range_pop if nvtx else (lambda: None)
        fork = torch.cuda.Event()
        fork.record(caller)
        main.wait_event(fork)
        self.side.wait_event(fork)
        # batches of more than 32 tokens with native weights: the shared expert's
        # down projection writes y_acc's starting value (no zero fill, no read
        # of the zeros), and the routed down projection waits for it
        store = (self.has_shared and not self.nvfp4 and not self.latent and T > 32)
        # bf16 decode batches: the router goes to the GPU ahead of the shared
        # expert's GEMV, whose CTAs would otherwise hold the registers that the
        # router's blocks wait for (1 % of the step, measured; with NVFP4
        # weights and at prefill the shared expert first is as fast or faster)
        route_first = not self.latent and not self.nvfp4 and T <= 32
        if route_first:
            push("route_permute")
            route_permute(self.c, x, self.w_router, self.bias, b.topk_idx, b.topk_w, b.ws,
                          stream=main)
            pop()
        if not store:
            # the accumulators start at zero on the side stream (beside the router)
            push("zero_acc")
            zero_acc(self.c, T, b.y_acc, stream=self.side)
            if self.latent:
                zero_acc(self.c_exp, T, b.y_lat_acc, stream=self.side)
            pop()
        zero = torch.cuda.Event()
        zero.record(self.side)

        # the shared expert runs on the side stream beside the routed path (at
        # decode it streams its weights while the router runs; at prefill its
        # GEMMs take the SMs the routing and permute kernels leave idle)
        if self.has_shared:
            push("shared")
            if self.nvfp4:
                shared_nvfp4(self.c, x, self.q4["shared_up"], self.q4["shared_down"], b.y_acc,
                             b.ws_shared, stream=self.side)
            elif store:
                shared_store(self.c, x, self.w_shared_up, self.w_shared_down, b.y_acc,
                             b.ws_shared, stream=self.side)
            else:
                shared(self.c, x, self.w_shared_up, self.w_shared_down, b.y_acc, b.ws_shared,
                       stream=self.side)
            pop()
        join = torch.cuda.Event()
        join.record(self.side)

        def shared_done():
            main.wait_event(join)

        if self.latent:
            out = self._forward_latent(x, b, main, zero, shared_done, partial, push, pop)
            self._join(caller, main)
            return out
        if not route_first:
            push("route_permute")
            route_permute(self.c, x, self.w_router, self.bias, b.topk_idx, b.topk_w, b.ws,
                          stream=main)
            pop()
        push("forward")
        if store:
            # y_acc holds the shared expert before the routed adds begin
            experts_up(self.c, x, self.w_up, b.ws, stream=main)
            shared_done()
            experts_down(self.c, T, self.w_down, b.ws, b.y_acc, stream=main)
        elif self.nvfp4:
            main.wait_event(zero)
            forward_nvfp4(self.c, x, self.q4["up"], self.q4["down"], b.ws, b.y_acc, stream=main)
        else:
            main.wait_event(zero)
            forward(self.c, x, self.w_up, self.w_down, b.ws, b.y_acc, stream=main)
        pop()
        shared_done()
        if not partial:
            push("finalize")
            finalize(self.c, T, b.y_acc, b.y, stream=main)
            pop()
        self._join(caller, main)
        return b.y_acc if partial else b.y

    @staticmethod
    def _join(caller, main):
        done = torch.cuda.Event()
        done.record(main)
        caller.wait_event(done)

    def _forward_latent(self, x, b, main, zero, shared_done, partial, push, pop):
        T = x.shape[0]
        push("route")
        route(self.c, x, self.w_router, self.bias, b.topk_idx, b.topk_w, b.ws_route, stream=main)
        pop()
        push("latent_in")
        latent_in(self.c, x, self.w_latent_fc1, b.x_lat, b.ws_lat, stream=main)
        pop()
        push("experts")
        ce = self.c_exp
        reset_status(b.ws, stream=main)
        permute(ce, b.x_lat, b.topk_idx, b.topk_w, b.ws, stream=main)
        main.wait_event(zero)
        if self.nvfp4:
            forward_nvfp4(ce, b.x_lat, self.q4["up"], self.q4["down"], b.ws, b.y_lat_acc,
                          stream=main)
        else:
            forward(ce, b.x_lat, self.w_up, self.w_down, b.ws, b.y_lat_acc, stream=main)
        finalize(ce, T, b.y_lat_acc, b.y_lat, stream=main)
        pop()
        shared_done()     # y_acc holds the shared expert before fc2 adds into it
        push("latent_out")
        latent_out(self.c, T, b.y_lat, self.w_latent_fc2, b.y_acc, b.ws_lat, stream=main)
        pop()
        if partial:
            return b.y_acc
        push("finalize")
        finalize(self.c, T, b.y_acc, b.y, stream=main)
        pop()
        return b.y

    def capture(self, T: int, slot: int = 0):
        """Capture the call sequence for T tokens in a CUDA graph (on the buffer set
        ``slot``).

        Returns (graph, x_static, y): write the input into ``x_static`` and
        ``graph.replay()`` writes ``y``."""
        g = self._graphs.get((T, slot))
        if g is None:
            x_static = torch.zeros((T, self.H), dtype=self.dtype, device=self.device)
            b = self.buffers(T, slot)
            s = torch.cuda.Stream(self.device)
            s.wait_stream(torch.cuda.current_stream(self.device))
            with torch.cuda.stream(s):           # warm up outside the graph
                self.forward(x_static, b)
            torch.cuda.current_stream(self.device).wait_stream(s)
            torch.cuda.synchronize(self.device)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                y = self.forward(x_static, b)
            g = (graph, x_static, y)
            self._graphs[(T, slot)] = g
        return g

    def pipeline(self, xs):
        """y for a sequence of host batches (pinned tensors [T, H], one T), with the
        host copies of one batch overlapping the block of another: the block runs
        as a CUDA graph on the current stream, host-to-device copies on one stream
        and device-to-host copies on another, over two buffer sets.  Every batch
        still has its own copy in and copy out.

        A generator: yields (index, y) in order, y a pinned host tensor [T, H] that
        stays valid until the generator is resumed twice more (it is reused for the
        batch after next); clone it to keep it."""
        xs = list(xs)
        if not xs:
            return
        T = xs[0].shape[0]
        dev = self.device
        comp = torch.cuda.current_stream(dev)
        if not hasattr(self, "_h2d"):
            with torch.cuda.device(dev):
                self._h2d = torch.cuda.Stream()
                self._d2h = torch.cuda.Stream()
        slots = []
        for s in (0, 1):
            graph, x_static, y = self.capture(T, s)
            key = ("pinned_out", T, s)
            yh = self._host.get(key)
            if yh is None:
                yh = torch.empty((T, self.H), dtype=self.dtype).pin_memory()
                self._host[key] = yh
            slots.append((graph, x_static, y, yh))
        in_free = [None, None]    # the slot's x_static was read by its last block call
        out_free = [None, None]   # the slot's y was copied out
        prev = None
        for i, xh in enumerate(xs):
            if xh.shape[0] != T:
                raise ValueError("pipeline: every batch needs the same token count")
            if not xh.is_pinned():
                raise ValueError("pipeline: host batches must be in pinned memory")
            graph, x_static, y, yh = slots[i % 2]
            if in_free[i % 2] is not None:
                self._h2d.wait_event(in_free[i % 2])
            with torch.cuda.stream(self._h2d):
                x_static.copy_(xh, non_blocking=True)
            copied = torch.cuda.Event()
            copied.record(self._h2d)
            comp.wait_event(copied)
            if out_free[i % 2] is not None:
                comp.wait_event(out_free[i % 2])
            graph.replay()
            done = torch.cuda.Event()
            done.record(comp)
            in_free[i % 2] = done
            self._d2h.wait_event(done)
            with torch.cuda.stream(self._d2h):
                yh.copy_(y, non_blocking=True)
            out = torch.cuda.Event()
            out.record(self._d2h)
            out_free[i % 2] = out
            if prev is not None:
                prev[1].synchronize()
                yield prev[0], prev[2]
            prev = (i, out, yh)
        prev[1].synchronize()
        yield prev[0], prev[2]

    def check(self, T: int) -> int:
        """Status word of the last call for T tokens (synchronises)."""
        b = self.buffers(T)
        rc = check_device(b.ws)
        for extra in (b.ws_shared, b.ws_route, b.ws_lat):
            if rc == 0 and extra is not None:
                rc = check_device(extra)
        return rc

    def __call__(self, x, use_graph: bool = True):
        """y = block(x).  A device tensor is computed in place on the current
        stream; a host tensor (or numpy array) goes through pinned staging
        buffers: host->device copy, the block (as a CUDA graph when
        ``use_graph``), device->host copy.

        Both forms return a buffer the block owns, like a CUDA graph's static
        output: the device y of ``forward`` for T tokens, or the pinned host
        output buffer for T tokens.  The next call with the same T overwrites
        it; clone the result to keep it."""
        if isinstance(x, torch.Tensor) and x.is_cuda:
            return self.forward(x)
        xh = _to_device(x, self.dtype, "cpu") if isinstance(x, np.ndarray) else x
        T = xh.shape[0]
        st = self._host.get(T)
        if st is None:
            st = (torch.empty((T, self.H), dtype=self.dtype).pin_memory(),
                  torch.empty((T, self.H), dtype=self.dtype).pin_memory())
            self._host[T] = st
        xin, yout = st
        if not xh.is_pinned():
            xin.copy_(xh)
            xh = xin
        if use_graph:
            graph, x_static, y = self.capture(T)
            x_static.copy_(xh, non_blocking=True)
            graph.replay()
        else:
            xd = xh.to(self.device, non_blocking=True)
            y = self.forward(xd)
        yout.copy_(y, non_blocking=True)
        torch.cuda.current_stream(self.device).synchronize()
        return yout
