"""The multi-rank host logic of bench.py on CPU: world_size-2 `gloo` ranks.

The benchmark runs independent replicas (one full step per rank, no data-path
collective); what crosses ranks is the barrier and the max-over-ranks step
time, and only rank 0 runs and prints the reference arm."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        # each rank times its own step; all report the slowest
        ms = bench.max_over_ranks(torch, dist, 1.5 + rank, torch.device("cpu"))
        rate = bench.whole_job_rate(1e9, world, ms)
        out.put((rank, ms, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rate_with_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, rate in res:
        assert ms == pytest.approx(2.5)                     # the slower rank's 1.5 + 1
        assert rate == pytest.approx(2 * 1e9 / 2.5e-3 / 1e9)


def test_reference_arm_runs_on_rank_zero_only():
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        warmup, steps, gpus = 1, 1, 2
    # a rank other than 0 returns at once, without touching the oracle
    assert bench.run_reference(Args, rank=1, world=2) is None


def test_every_profiled_row_has_a_committed_summary():
    """The bench reads a row's DRAM traffic from its committed ncu summary; each
    mapped file must exist, carry its command and parse to a positive number."""
    sys.path.insert(0, ROOT)
    import bench
    for row, fname in bench.PROFILE_OF_ROW.items():
        path = os.path.join(ROOT, "profiles", fname)
        assert os.path.exists(path), (row, fname)
        text = open(path).read()
        assert "ncu " in text and "--clock-control none" in text, fname
        t = bench.profiled_traffic(row)
        assert t is not None and t > 0, (row, fname)
