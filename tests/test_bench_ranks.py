"""The multi-replica bookkeeping of bench.py on CPU: two gloo ranks, the barrier and the max-over-ranks
reduction every reported time goes through, and the whole-job throughput."""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r = bench.Ranks(world, torch.device("cpu"))
        r.barrier()
        slowest = r.max(1.0 + rank * 0.25)  # rank 1 is the slower one
        r.barrier()
        out.put((rank, slowest))
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, port = 2, _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(world))
    assert got == {0: 1.25, 1: 1.25}


def test_single_rank_and_job_throughput():
    r = bench.Ranks(1)
    r.barrier()
    assert r.max(3.5) == 3.5
    assert bench.job_throughput(1, 0.002) == 500.0
    assert bench.job_throughput(8, 0.002) == 4000.0  # weak scaling: every replica runs whole steps
