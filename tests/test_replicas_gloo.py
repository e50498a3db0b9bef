"""The N > 1 path of bench.py (replicas only): each rank times its own copy of the
workload, the job's time is the max over ranks and the throughput counts every rank's
units. Exercised with two gloo ranks on the CPU (the data path has no collective)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r timed (10 + r) ms per step and (200 - r) ms of prefill
        ms_step, prefill_ms = bench.max_over_ranks([10.0 + rank, 200.0 - rank])
        value = bench.replica_throughput(1, world, ms_step)
        q.put((rank, ms_step, prefill_ms, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms_step, prefill_ms, value in out:
        assert ms_step == 11.0 and prefill_ms == 200.0  # the slowest rank's times, on every rank
        assert value == pytest.approx(2 / 11e-3)          # both ranks' tokens over the slowest time


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert not dist.is_initialized()
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert bench.replica_throughput(4096, 1, 200.0) == pytest.approx(20480.0)
