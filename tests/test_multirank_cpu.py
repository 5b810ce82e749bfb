"""The multi-GPU path is replicas only (no data-path collective): each rank runs
the whole workload and rank 0 reports all ranks' FLOPs over the slowest rank's
time.  These world-size-2 gloo tests check that host logic on the CPU."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        # Each rank's own "total timed ms"; rank 1 is the slower one.
        mine = 100.0 + 50.0 * rank
        slowest = bench.max_over_ranks(mine, world, device="cpu")
        bench.barrier(world)
        value = bench.whole_job_tflops(1e12, 10, world, slowest)
        q.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_replicas_report_slowest_rank_and_all_flops():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    results = sorted(q.get(timeout=10) for _ in range(world))
    for rank, slowest, value in results:
        assert slowest == 150.0  # max over ranks, on every rank
        # 2 ranks x 1e12 FLOP x 10 steps in 0.150 s
        assert value == pytest.approx(2 * 1e12 * 10 / 0.150 / 1e12)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_tflops(2e12, 5, 1, 1000.0) == pytest.approx(10.0)
