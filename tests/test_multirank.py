"""The multi-GPU mode of bench.py is N independent replicas of the step
(the path has no exchange step). Its host-side logic -- the time taken as the
maximum over ranks and the whole-job throughput -- runs here as two gloo
ranks on the CPU."""

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


def _worker(rank, world, port, times, q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank], world, torch.device("cpu"))
        q.put((rank, ms, bench.job_gbs(world, 10, ms)))
    finally:
        dist.destroy_process_group()


def test_replicas_take_the_slowest_rank():
    import bench
    world, port = 2, _free_port()
    times = [12.5, 20.0]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, gbs in res:
        assert ms == max(times)
        # two replicas of the step in the slowest rank's time
        assert gbs == pytest.approx(2 * bench.STEP_BYTES * 10 / (max(times) * 1e-3) / 1e9)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(7.0, 1, torch.device("cpu")) == 7.0
    assert bench.job_gbs(1, 4, 2.0) == pytest.approx(bench.STEP_BYTES * 4 / 2e-3 / 1e9)
