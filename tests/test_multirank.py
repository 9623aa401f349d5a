"""The benchmark's multi-rank path on CPU: two gloo ranks.

Token data parallelism has no data-path collective; what the ranks share is
the bookkeeping: disjoint input batches per rank, one step count for all
ranks, the max-over-ranks time of the timed region, and the whole-job
throughput computed from it.  The
reference arm runs on rank 0 only.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = 100.0 + 25.0 * rank            # rank 1 is the slow one
        mx = bench.max_over_ranks(elapsed, dist, torch.device("cpu"))
        ids = bench.rank_batch_ids(4, rank)
        steps = bench.agree_steps(100 + 7 * rank, dist, torch.device("cpu"))
        gathered = [None] * world
        dist.all_gather_object(gathered, ids)
        q.put((rank, mx, gathered, steps))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_bookkeeping():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, gathered, steps in out:
        assert mx == 125.0                        # every rank sees the slowest rank's time
        assert steps == 100                       # every rank times rank 0's step count
        flat = [i for ids in gathered for i in ids]
        assert len(flat) == len(set(flat)) == 8   # batches are disjoint across ranks
    # whole-job throughput: all ranks' tokens over the max time
    assert bench.job_throughput(8, world, 100, 125.0) == pytest.approx(8 * 2 * 100 / 0.125)


def test_reference_arm_runs_on_rank_zero_only():
    class A:
        workload = "tiny_f32_t64"
        set = []
        warmup = 0
        steps = 1
    assert bench.run_reference(A(), rank=1, world=2) is None
    out = bench.run_reference(A(), rank=0, world=2)
    assert out["impl"] == "reference" and out["value"] > 0
    assert out["e2e"]["h2d_bytes_per_step"] == 0
