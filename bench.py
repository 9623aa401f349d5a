"""Benchmark of the Nemotron-H non-gated MoE block forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--no-cpu-baseline]

One step = one whole block call (router, permute, routed up/down experts,
shared expert on a second stream, finalize) over one batch of T seeded
synthetic tokens, replayed as a CUDA graph with weights and inputs resident
in HBM.  The timed region holds exactly K steps between two barriers +
device synchronisations and is measured with CUDA events; with N GPUs
(torchrun) every rank runs its own batch (token data parallelism: no
collective on the data path) and the max over ranks is reported.

Rank 0 prints one JSON line with the throughput (tokens/s), the TFLOP/s and
roofline fractions, the dominant kernel's roofline (CUDA-event timed), the
end-to-end throughput through the public host API, the oracle's CPU
throughput on a bounded sample, and the SM clocks sampled during the timed
region.  ``--impl reference`` times the fp64 CPU oracle on the same workload
(rank 0 only) and prints the same line with ``"impl": "reference"``.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE-block tokens/s and TFLOP/s (frac of bf16 peak / HBM roofline), 1×B200"
DEFAULT_WORKLOAD = "prefill_bf16_t16384"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCE_DIR = "non_gated_relu_b200/csrc"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=0, help="timed steps (0: about 2 s of work)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=synth.CONFIG_ORDER)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--parallel", default="dp", choices=["dp", "tp"],
                    help="dp: disjoint token batches per GPU, replicated weights (weak "
                         "scaling); tp: I and S sharded over the GPUs, same tokens, one "
                         "all-reduce of y per step (strong scaling)")
    ap.add_argument("--batches", type=int, default=4, help="distinct input batches cycled")
    ap.add_argument("--eager", action="store_true",
                    help="timed loop calls the block eagerly (NVTX range per call) instead of "
                         "replaying CUDA graphs")
    ap.add_argument("--only-timed", action="store_true",
                    help="run the timed loop only (inside an NVTX range 'timed'), for profilers")
    ap.add_argument("--set", action="append", default=[], metavar="KEY=VALUE",
                    help="override a workload field (smaller profiling cases of the same kernels)")
    return ap.parse_args()


def workload(args):
    cfg = synth.CONFIGS[args.workload]
    kw = {}
    for item in args.set:
        k, v = item.split("=", 1)
        cur = getattr(cfg, k)
        kw[k] = type(cur)(v) if not isinstance(cur, bool) else v.lower() in ("1", "true")
    return cfg.replace(**kw) if kw else cfg


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def skew_b(cfg):
    if not cfg.skew_hot_groups:
        return None
    with open(os.path.join(ROOT, "tests", "golden", "skew_prefill_t2048.json")) as f:
        return json.load(f)["b"]


def batch_x(cfg, i):
    """Input batch i: batch 0 is the workload's own x; others use seed offsets."""
    c = cfg if i == 0 else cfg.replace(seed=cfg.seed + 1000 * i)
    x, _, _, _, _ = synth.make_router_and_x(c, skew_b(cfg))
    return x


def rank_batch_ids(nb, rank):
    """Input batches of one rank: every rank gets its own nb batches (token data
    parallelism: ranks never share a batch); rank 0's first batch is the
    workload's own x."""
    return [rank * nb + i for i in range(nb)]


def max_over_ranks(elapsed_ms, dist, device):
    """Timed-region length of the whole job: the slowest rank's (all-reduce MAX)."""
    if dist is None:
        return float(elapsed_ms)
    import torch
    t = torch.tensor([float(elapsed_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def agree_steps(steps, dist, device):
    """Rank 0's step count on every rank, so that all ranks time the same work
    and take the same collective steps."""
    if dist is None:
        return int(steps)
    import torch
    t = torch.tensor([int(steps)], dtype=torch.int64, device=device)
    dist.broadcast(t, 0)
    return int(t.item())


def job_throughput(tokens_per_rank_step, world, steps, elapsed_ms):
    """Whole-job tokens/s: the tokens all ranks processed over the max-over-ranks time."""
    return tokens_per_rank_step * world * steps / (elapsed_ms / 1e3)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        # nvidia-smi numbers GPUs physically; under CUDA_VISIBLE_DEVICES the
        # torch index differs, so address the device by its UUID when known
        self.idx = str(gpu_index)
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(gpu_index).uuid)
            if uuid:
                self.idx = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            pass
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [v.strip() for v in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU oracle
def host_cores():
    """CPU cores this process may run on (affinity mask; os.cpu_count() without one)."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def oracle_rate(inp, budget_s=8.0, threads=1):
    """Oracle tokens/s on a bounded sample: rounds of `threads` independent
    single-threaded fp64 C calls, one token shard each (ctypes releases the
    GIL), repeated until `budget_s` has passed.  Tokens are independent, so the
    cost is linear in the token count."""
    import oracle
    cfg = inp.cfg
    n = min(cfg.T, max(8, threads))
    tok = np.arange(n, dtype=np.int64)
    done, t0 = 0, time.perf_counter()
    while True:
        oracle.forward_parallel(inp, tokens=tok, threads=threads)
        done += n
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return done / el, done, el


def cpu_baseline(inp):
    """The oracle on this host: all usable cores (one token shard per thread)
    and, for comparison, one core."""
    cores = host_cores()
    r1, n1, e1 = oracle_rate(inp, threads=1)
    rn, nn, en = oracle_rate(inp, threads=cores) if cores > 1 else (r1, n1, e1)
    n = min(inp.cfg.T, max(8, cores))
    return {"value": round(rn, 4), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "host_cores": os.cpu_count(),
            "sample": (f"first {n} tokens of the batch split over {cores} threads, repeated: "
                       f"{nn} tokens in {en:.1f} s, fp64 C oracle"),
            "single_core": {"value": round(r1, 4), "unit": "tokens/s",
                            "sample": f"first {min(inp.cfg.T, 8)} tokens, repeated: {n1} tokens "
                                      f"in {e1:.1f} s on one thread"}}


# ----------------------------------------------------------------------------- ours
def run_ours(args, rank, world, local_rank):
    import torch
    import non_gated_relu_b200 as nh

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = workload(args)
    inp = synth.make_inputs(cfg, skew_b=skew_b(cfg))
    blk = nh.NemotronHMoE(cfg, inp.w_router, inp.w_up, inp.w_down, inp.w_shared_up,
                          inp.w_shared_down, device=dev, nvfp4=inp.nvfp4,
                          w_latent_fc1=inp.w_latent_fc1, w_latent_fc2=inp.w_latent_fc2)
    T = cfg.T
    nb = max(1, args.batches)
    xs = []
    for i in rank_batch_ids(nb, rank):
        xi = inp.x if i == 0 else batch_x(cfg, i)
        t = torch.from_numpy(xi)
        t = t.view(torch.bfloat16) if xi.dtype == np.uint16 else t
        xs.append(t.to(dev))
    # one graph per input batch (buffers shared: the replays are stream-ordered)
    graphs = []
    b = blk.buffers(T)
    for i in range(nb):
        s = torch.cuda.Stream(dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            blk.forward(xs[i], b)
        torch.cuda.current_stream(dev).wait_stream(s)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            blk.forward(xs[i], b)
        graphs.append(g)
    rc = blk.check(T)
    if rc != 0:
        raise RuntimeError(f"device status {rc} after warm-up")

    main = torch.cuda.current_stream(dev)
    for i in range(max(3, args.warmup)):
        graphs[i % nb].replay()
    torch.cuda.synchronize(dev)

    # step-time estimate -> default number of steps (about 2 s timed)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for i in range(20):
        graphs[i % nb].replay()
    e1.record(main)
    e1.synchronize()
    est = e0.elapsed_time(e1) / 20.0
    steps = args.steps if args.steps > 0 else int(max(20, min(20000, 2000.0 / max(est, 1e-3))))

    dist = None
    if world > 1:
        import torch.distributed as dist
    steps = agree_steps(steps, dist, dev)
    clocks = ClockSampler(local_rank)
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed")
    t_start.record(main)
    if args.eager:
        for i in range(steps):
            blk.forward(xs[i % nb], b, nvtx=True)
    else:
        for i in range(steps):
            graphs[i % nb].replay()
    t_end.record(main)
    torch.cuda.synchronize(dev)
    torch.cuda.nvtx.range_pop()
    if dist:
        dist.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    clk = clocks.stop() if rank == 0 else None
    elapsed_ms = max_over_ranks(elapsed_ms, dist, dev)
    rc = blk.check(T)
    if rc != 0:
        raise RuntimeError(f"device status {rc} after the timed region")
    if args.only_timed:
        if rank == 0:
            return {"workload": cfg.name, "T": T, "E": cfg.E, "steps": steps,
                    "ms_per_step": round(elapsed_ms / steps, 5), "only_timed": True}
        return None

    # per-kernel durations (eager calls, events on the launching streams)
    ksteps = min(steps, 200)
    kern = kernel_times(blk, xs, b, nb, steps=ksteps)
    # distinct routed experts of every input batch (the bytes a decode step
    # must stream depend on them); averaged below with each batch's share of
    # the timed steps and of the kernel-timing calls
    ds = []
    for i in range(nb):
        blk.forward(xs[i], b)
        torch.cuda.synchronize(dev)
        ds.append(distinct_experts(cfg, blk.buffers(T).topk_idx.cpu().numpy()))

    # end to end through the public host API: every step copies its batch in from
    # pinned host memory and its result out to pinned host memory; the block's
    # pipelined host call overlaps one step's copies with another step's block
    xh = [x.cpu().pin_memory() for x in xs]
    for _ in blk.pipeline([xh[i % nb] for i in range(4)]):
        pass
    e2e_steps = min(steps, 2000)
    torch.cuda.synchronize(dev)
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0.record(main)
    for _ in blk.pipeline([xh[i % nb] for i in range(e2e_steps)]):
        pass
    h1.record(blk._d2h)        # after the last device-to-host copy
    torch.cuda.synchronize(dev)
    e2e_total_ms = max_over_ranks(h0.elapsed_time(h1), dist, dev)
    e2e_ms = e2e_total_ms / e2e_steps

    result = None
    if rank == 0:
        result = report(args, cfg, inp, world, steps, elapsed_ms, clk, kern, e2e_ms, blk, ds,
                        ksteps)
    if dist:
        dist.barrier()
    del graphs
    return result


def kernel_times(blk, xs, b, nb, steps):
    """Average CUDA-event duration of each phase of the block, eager, on its stream."""
    import torch
    import non_gated_relu_b200 as nh
    main = torch.cuda.current_stream(blk.device)
    T = xs[0].shape[0]
    names = ["zero_acc", "route", "permute", "experts_up", "experts_down", "shared", "finalize"]
    # decode batches (T <= 32, bf16 or NVFP4 experts): nh_moe_forward[_nvfp4]
    # runs the up and down projections as one launch
    fused = T <= 32 and (blk.nvfp4 or blk.cfg.dtype == "bf16")
    store = blk.has_shared and not blk.nvfp4 and not blk.latent and T > 32
    acc = {n: 0.0 for n in names}
    ev = {n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for n in names}
    for i in range(steps):
        x = xs[i % nb]
        def timed(n, fn, stream=main):
            ev[n][0].record(stream)
            fn()
            ev[n][1].record(stream)
        if blk.latent:
            timed("zero_acc", lambda: (nh.zero_acc(blk.c, T, b.y_acc, stream=main),
                                       nh.zero_acc(blk.c_exp, T, b.y_lat_acc, stream=main)))
        elif not store:
            timed("zero_acc", lambda: nh.zero_acc(blk.c, T, b.y_acc, stream=main))
        if store:
            # the block's schedule for these batches: the shared expert writes
            # y_acc's starting value, no zero fill
            timed("shared", lambda: nh.shared_store(blk.c, x, blk.w_shared_up, blk.w_shared_down,
                                                     b.y_acc, b.ws_shared, stream=main))
        elif blk.has_shared and blk.nvfp4:
            timed("shared", lambda: nh.shared_nvfp4(blk.c, x, blk.q4["shared_up"],
                                                     blk.q4["shared_down"], b.y_acc,
                                                     b.ws_shared, stream=main))
        elif blk.has_shared:
            timed("shared", lambda: nh.shared(blk.c, x, blk.w_shared_up, blk.w_shared_down,
                                               b.y_acc, b.ws_shared, stream=main))
        if blk.latent:
            # routing on x, fc1 (counted with the permute), experts in width L
            ce = blk.c_exp
            timed("route", lambda: nh.route(blk.c, x, blk.w_router, blk.bias, b.topk_idx,
                                             b.topk_w, b.ws_route, stream=main))
            timed("permute", lambda: (nh.latent_in(blk.c, x, blk.w_latent_fc1, b.x_lat, b.ws_lat,
                                                   stream=main),
                                      nh.reset_status(b.ws, stream=main),
                                      nh.permute(ce, b.x_lat, b.topk_idx, b.topk_w, b.ws,
                                                 stream=main)))
            xe, yacc = b.x_lat, b.y_lat_acc
        else:
            ce = blk.c
            timed("route", lambda: nh.route(blk.c, x, blk.w_router, blk.bias, b.topk_idx,
                                             b.topk_w, b.ws, stream=main))
            timed("permute", lambda: nh.permute(blk.c, x, b.topk_idx, b.topk_w, b.ws, stream=main))
            xe, yacc = x, b.y_acc
        if blk.nvfp4 and not blk.latent:
            # up and down run back to back in one call; each is timed as half
            timed("experts_up", lambda: nh.forward_nvfp4(blk.c, x, blk.q4["up"], blk.q4["down"],
                                                          b.ws, yacc, stream=main))
        elif fused and not blk.nvfp4:
            # decode: nh_moe_forward runs both projections as one launch
            timed("experts_up", lambda: nh.forward(ce, xe, blk.w_up, blk.w_down, b.ws, yacc,
                                                    stream=main))
        else:
            timed("experts_up", lambda: nh.experts_up(ce, xe, blk.w_up, b.ws, stream=main))
            timed("experts_down", lambda: nh.experts_down(ce, T, blk.w_down, b.ws, yacc,
                                                           stream=main))
        if blk.latent:
            # routed sum rounded in width L, fc2 onto y_acc, the one rounding
            timed("finalize", lambda: (nh.finalize(ce, T, b.y_lat_acc, b.y_lat, stream=main),
                                       nh.latent_out(blk.c, T, b.y_lat, blk.w_latent_fc2,
                                                     b.y_acc, b.ws_lat, stream=main),
                                       nh.finalize(blk.c, T, b.y_acc, b.y, stream=main)))
        else:
            timed("finalize", lambda: nh.finalize(blk.c, T, b.y_acc, b.y, stream=main))
        torch.cuda.synchronize(blk.device)
        for n in names:
            if ((n == "shared" and not blk.has_shared) or (n == "zero_acc" and store) or
                    (n == "experts_down" and (blk.nvfp4 or fused))):
                continue
            acc[n] += ev[n][0].elapsed_time(ev[n][1])
    out = {n: acc[n] / steps for n in names}
    if blk.nvfp4 or fused:
        out["experts_up"] = out["experts_down"] = acc["experts_up"] / steps / 2
    if fused:
        out["experts_fused"] = acc["experts_up"] / steps
    return out


def launches_per_step(cfg):
    """Kernels of one block call (memsets excluded), as nh_moe.cu launches them."""
    T = cfg.T
    # routed up and down: one launch for decode batches (bf16 or NVFP4 experts)
    experts = 1 if T <= 32 and (cfg.dtype == "bf16" or cfg.weight_format == "nvfp4") else 2
    shared = 2 if cfg.n_shared_experts else 0
    if getattr(cfg, "latent_size", 0):
        # route, fc1, permute, experts, finalize of the latent sum, fc2, cast, shared
        n = 1 if T <= 32 else (3 if cfg.dtype == "bf16" and cfg.E % 32 == 0 else 2)
        n += 1 + (1 if T <= 256 else 4) + experts + 1 + 1 + 1
        return n + shared
    if T <= 32:
        n = 1                                   # router and permute in one launch
    else:
        if cfg.dtype == "bf16" and cfg.E % 32 == 0:
            n = 3                               # weight split, tensor-core logits, select
        else:
            n = 2                               # logits, select
        n += 1 if T <= 256 else 4               # permute (one block, or hist/scan/scatter/gather)
    return n + experts + shared + 1             # + finalize


def distinct_experts(cfg, idx):
    return int(len(np.unique(idx)))


def cycled_mean(values, steps):
    """Mean of per-batch values over `steps` calls that cycle through the batches."""
    nb = len(values)
    counts = [len(range(i, steps, nb)) for i in range(nb)]
    return float(np.dot(values, counts) / sum(counts))


def report(args, cfg, inp, world, steps, elapsed_ms, clk, kern, e2e_ms, blk, ds, ksteps):
    pk, pk_kind = peaks()
    burst = pk["bf16_tflops"]
    sustained = pk.get("bf16_tflops_sustained") or burst
    T = cfg.T
    ms = elapsed_ms / steps
    value = job_throughput(T, world, steps, elapsed_ms)
    flops_tok = cfg.flops_per_token()
    tflops = flops_tok * T * world / (ms / 1e3) / 1e12
    elem = 2 if cfg.dtype == "bf16" else 4
    welem = 0.5 + 1.0 / 16 if cfg.weight_format == "nvfp4" else elem   # bytes per weight
    expert_bytes = int(cfg.I * cfg.HE * welem)     # one projection of one expert
    shared_bytes = int(2 * cfg.S * cfg.H * welem) if cfg.n_shared_experts else 0
    rows = T * cfg.k
    # algorithmic bytes of one step: touched weights + router + x in + y out,
    # with D (distinct experts) averaged over the batches the timed steps cycle
    latent_bytes = 2 * cfg.latent_size * cfg.H * elem if cfg.latent_size else 0
    fixed_bytes = shared_bytes + latent_bytes + cfg.E * cfg.H * 4 + 2 * T * cfg.H * elem
    d_step = cycled_mean(ds, steps)
    step_bytes = d_step * 2 * expert_bytes + fixed_bytes
    hbm_step = step_bytes / (ms / 1e3) / 1e9
    # dominant kernel roofline: its mean CUDA-event duration, timed alone
    # (eager), against the burst peaks
    decode = T <= 64
    dom = "experts_up" if kern["experts_up"] >= kern["experts_down"] else "experts_down"
    if "experts_fused" in kern:
        dom = "experts_fused"
    if decode:
        d_kern = cycled_mean(ds, ksteps)
        kb = d_kern * expert_bytes + rows * (cfg.HE + cfg.I) * elem
        if dom == "experts_fused":
            kb *= 2          # both projections in the launch
        ach = kb / (kern[dom] / 1e3) / 1e9
        peak = pk["hbm_gbs"]
        roof = {"bound": "hbm", "kernel": dom, "achieved": round(ach, 1), "peak": peak,
                "unit": "GB/s", "frac": round(ach / peak, 4), "peak_kind": pk_kind,
                "algorithmic_bytes_per_launch": int(round(kb)),
                "distinct_experts_per_launch": round(d_kern, 3),
                "ms_per_launch": round(kern[dom], 5)}
    else:
        kf = 2.0 * rows * cfg.HE * cfg.I
        ach = kf / (kern[dom] / 1e3) / 1e12
        roof = {"bound": "tensor", "kernel": dom, "achieved": round(ach, 1), "peak": burst,
                "unit": "TFLOP/s", "frac": round(ach / burst, 4),
                "peak_kind": pk_kind + " burst (kernel timed alone)",
                "algorithmic_flops_per_launch": kf, "ms_per_launch": round(kern[dom], 5)}
    roof["traffic"] = ncu_traffic(args.workload, roof["kernel"])
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world,
        "steps": steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("nvfp4 weights, bf16 activations" if cfg.weight_format == "nvfp4"
                  else ("bf16" if cfg.dtype == "bf16" else "f32")), "data": "synthetic",
        "config": {"workload": cfg.name, "tokens_per_step_per_gpu": T, "hidden_size": cfg.H,
                   "n_routed_experts": cfg.E, "n_group": cfg.G, "topk_group": cfg.tg,
                   "num_experts_per_tok": cfg.k, "moe_intermediate_size": cfg.I,
                   "moe_shared_expert_intermediate_size": cfg.S,
                   "parallelism": f"dp{world} (token batches, replicated weights)",
                   "input_batches_cycled": args.batches,
                   "l2": (f"inputs larger than L2: {step_bytes / 1e6:.0f} MB of weights and "
                          f"activations touched per step (mean over the cycled batches)")},
        "tflops": round(tflops, 3),
        # whole step: the burst peak, and the sustained (seconds-long, power-capped) one
        "tflops_frac": round(tflops / burst, 4),
        "tflops_frac_sustained": round(tflops / sustained, 4),
        "hbm_gbs_step": round(hbm_step, 1), "hbm_frac_step": round(hbm_step / pk["hbm_gbs"], 4),
        "distinct_experts_per_batch": ds,
        "roofline": roof,
        "kernel_ms": {k: round(v, 5) for k, v in kern.items()},
        "e2e": {"value": round(job_throughput(T, world, 1, e2e_ms), 2), "unit": "tokens/s",
                "ms_per_step": round(e2e_ms, 5),
                "h2d_bytes_per_step": T * cfg.H * elem, "d2h_bytes_per_step": T * cfg.H * elem},
        "gpu_launches": launches_per_step(cfg) * steps,
        "clocks": clk,
        "peaks": {"kind": pk_kind, "hbm_gbs": pk["hbm_gbs"], "bf16_tflops": burst,
                  "bf16_tflops_sustained": pk.get("bf16_tflops_sustained")},
    }
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(inp)
    return out


def run_tp(args, rank, world, local_rank):
    """Tensor parallel: every rank holds its 64-feature blocks of I and S, all
    ranks process the same T tokens, and one NCCL all-reduce sums the float32
    block output per step (non_gated_relu_b200.tp).  The rank's own path runs
    as a CUDA graph; the all-reduce and the final rounding follow it on the
    same stream.  value = T / step time (strong scaling)."""
    import torch
    from non_gated_relu_b200 import tp

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = workload(args)
    inp = synth.make_inputs(cfg, skew_b=skew_b(cfg))
    blk = tp.TPNemotronHMoE(cfg, inp.w_router, inp.w_up, inp.w_down, inp.w_shared_up,
                            inp.w_shared_down, nvfp4=inp.nvfp4, world=world, rank=rank,
                            device=dev)
    T = cfg.T
    nb = max(1, args.batches)
    xs = []
    for i in range(nb):                          # the same batches on every rank
        xi = inp.x if i == 0 else batch_x(cfg, i)
        t = torch.from_numpy(xi)
        t = t.view(torch.bfloat16) if xi.dtype == np.uint16 else t
        xs.append(t.to(dev))
    b = blk.block.buffers(T)
    graphs = []
    for i in range(nb):
        s = torch.cuda.Stream(dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            blk.partial(xs[i])
        torch.cuda.current_stream(dev).wait_stream(s)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            blk.partial(xs[i])
        graphs.append(g)

    def step(i):
        graphs[i % nb].replay()
        tp.all_reduce_sum(b.y_acc)
        return blk.output(b.y_acc)

    main = torch.cuda.current_stream(dev)
    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for i in range(20):
        step(i)
    e1.record(main)
    e1.synchronize()
    est = e0.elapsed_time(e1) / 20.0
    steps = args.steps if args.steps > 0 else int(max(20, min(20000, 2000.0 / max(est, 1e-3))))
    if world > 1:
        import torch.distributed as dist
        dist_mod = dist
        # every rank runs the same number of steps (and so the same collectives)
        steps = agree_steps(steps, dist, dev)
    else:
        dist_mod = None
    clocks = ClockSampler(local_rank)
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    if dist_mod:
        dist_mod.barrier()
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(main)
    for i in range(steps):
        step(i)
    t1.record(main)
    torch.cuda.synchronize(dev)
    if dist_mod:
        dist_mod.barrier()
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), dist_mod, dev)
    clk = clocks.stop() if rank == 0 else None
    rc = blk.block.check(T)
    if rc != 0:
        raise RuntimeError(f"device status {rc} after the timed region")
    # end to end: pinned host x -> device -> step -> host y, every step
    xh = [x.cpu().pin_memory() for x in xs]
    xd = torch.empty_like(xs[0])
    yh = torch.empty((T, cfg.H), dtype=xs[0].dtype).pin_memory()
    e2e_steps = min(steps, 2000)

    def e2e_step(i):
        xd.copy_(xh[i % nb], non_blocking=True)
        blk.partial(xd)
        tp.all_reduce_sum(b.y_acc)
        yh.copy_(blk.output(b.y_acc), non_blocking=True)
        main.synchronize()
    for i in range(3):
        e2e_step(i)
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0.record(main)
    for i in range(e2e_steps):
        e2e_step(i)
    h1.record(main)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(h0.elapsed_time(h1), dist_mod, dev) / e2e_steps
    del graphs
    if rank != 0:
        return None
    ms = elapsed_ms / steps
    elem = 2 if cfg.dtype == "bf16" else 4
    return {
        "metric": METRIC, "value": round(T / (ms / 1e3), 2), "unit": "tokens/s",
        "n_gpus": world, "steps": steps, "warmup": max(3, args.warmup),
        "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None,
        "dtype": ("nvfp4 weights, bf16 activations" if cfg.weight_format == "nvfp4"
                  else ("bf16" if cfg.dtype == "bf16" else "f32")), "data": "synthetic",
        "config": {"workload": cfg.name, "tokens_per_step": T,
                   "parallelism": f"tp{world} (I and S in 64-feature blocks per GPU, one "
                                  f"all-reduce of the float32 block output per step)",
                   "moe_intermediate_size_per_gpu": blk.cfg_rank.moe_intermediate_size,
                   "moe_shared_expert_intermediate_size_per_gpu":
                       blk.cfg_rank.moe_shared_expert_intermediate_size,
                   "l2": "inputs larger than L2 (the expert weights touched per step)"},
        "e2e": {"value": round(T / (e2e_ms / 1e3), 2), "unit": "tokens/s",
                "ms_per_step": round(e2e_ms, 5),
                "h2d_bytes_per_step": T * cfg.H * elem, "d2h_bytes_per_step": T * cfg.H * elem},
        "gpu_launches": (launches_per_step(blk.cfg_rank) + 1) * steps,
        "clocks": clk,
    }


def kernel_hash():
    """Hash of every CUDA source of the library: profiler counters recorded for
    one build are reported only while the sources are unchanged."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, KERNEL_SOURCE_DIR)
    for name in sorted(os.listdir(d)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(d, name), "rb") as f:
                h.update(name.encode())
                h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload, kernel):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel sources changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    rec = d.get(workload, {}).get(kernel)
    if not rec or rec.get("kernel_hash") != kernel_hash():
        return None
    return rec.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- reference
def run_reference(args, rank, world):
    """The fp64 CPU oracle on this host's cores: each step runs the whole block
    on a bounded sample of the workload's tokens, one token shard per core
    (independent single-threaded C calls; tokens are independent)."""
    if rank != 0:
        return None
    cfg = workload(args)
    import oracle
    inp = synth.make_inputs(cfg, skew_b=skew_b(cfg))
    cores = host_cores()
    n = min(cfg.T, max(8, cores))
    tok = np.arange(n, dtype=np.int64)
    for _ in range(max(0, min(args.warmup, 1))):
        oracle.forward_parallel(inp, tokens=tok, threads=cores)
    steps = args.steps if args.steps > 0 else 10
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle.forward_parallel(inp, tokens=tok, threads=cores)
    el = time.perf_counter() - t0
    value = n * steps / el
    return {"metric": METRIC, "impl": "reference", "value": round(value, 4), "unit": "tokens/s",
            "n_gpus": world, "steps": steps, "warmup": args.warmup,
            "ms_per_step": round(el / steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "tokens_per_step_per_gpu": cfg.T,
                       "sample_tokens_per_step": n},
            "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "host_cores": os.cpu_count(),
                             "sample": f"{n} tokens per step (the first {n} of the batch) "
                                       f"split over {cores} threads, fp64 C oracle"},
            "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return 0
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        out = (run_tp if args.parallel == "tp" else run_ours)(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank == 0 and out is not None:
        print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
