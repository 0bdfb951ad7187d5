"""CPU checks of bench.py's N > 1 path (replicas): two gloo ranks run the
same collectives the GPU ranks run over NCCL -- the barrier and the maximum
of the per-rank time -- and the whole-job rate counts every rank's work over
the slowest rank's time.  Under torchrun the reference arm runs on rank 0
only; the other ranks exit 0 without output."""
from __future__ import annotations

import os
import socket
import subprocess
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        barrier, max_over_ranks = bench.replica_collectives(world, torch.device("cpu"))
        barrier()
        t = max_over_ranks(0.25 + 0.5 * rank)  # rank 1 is the slow one
        barrier()
        out.put((rank, t, bench.whole_job_tops(2e12, 10, world, t)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, tops in got:
        assert t == 0.75  # every rank sees the slowest rank's time
        assert abs(tops - 2e12 * 10 * 2 / 0.75 / 1e12) < 1e-9


def test_single_rank_needs_no_process_group():
    import bench
    barrier, max_over_ranks = bench.replica_collectives(1, torch.device("cpu"))
    barrier()
    assert max_over_ranks(1.5) == 1.5
    assert bench.whole_job_tops(1e12, 4, 1, 2.0) == 2.0


def test_reference_arm_only_on_rank_zero():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
