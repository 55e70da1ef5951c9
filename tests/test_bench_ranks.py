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


def test_gpus_flag_starts_the_replicas_itself():
    """`bench.py --gpus 2` without a launcher starts two ranks (torchrun, one process per GPU) and the line
    reports both: n_gpus 2, the slowest rank's step time, the whole-job rate."""
    import json
    import subprocess
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--replica-dry-run",
                        "--steps", "3", "--warmup", "3", "--config", "tiny"], capture_output=True, text=True,
                       timeout=240, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout  # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["config"]["parallelism"] == "replicas x2"
    assert d["ms_per_step"] == 2.0 and d["value"] == 1000.0  # max over ranks (rank 1: 2 ms), 2 replicas


def test_replica_command_and_world_mismatch(monkeypatch):
    cmd = bench.replica_command(["--gpus", "4", "--steps", "5"], 4, 29500)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert cmd[cmd.index("--nproc-per-node") + 1] == "4" and cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-4:] == ["--gpus", "4", "--steps", "5"]
    monkeypatch.setenv("WORLD_SIZE", "2")
    import pytest
    with pytest.raises(SystemExit):
        bench.main(["--gpus", "4", "--replica-dry-run", "--config", "tiny"])
