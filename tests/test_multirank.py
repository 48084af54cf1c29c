"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2): the max-over-ranks timing
reduction, the whole-job rate for independent replicas, and the reference arm's rank handling."""
from __future__ import annotations

import os
import socket
import subprocess
import sys
from datetime import timedelta

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    elapsed = 10.0 + 5.0 * rank                      # rank 1 is the slower one
    m = bench.reduce_max(elapsed, world, "cpu")
    rate = bench.whole_job_rate(131072, 10, world, m)
    dist.barrier()
    out.put((rank, m, rate))
    dist.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_time():
    ctx = mp.get_context("spawn")
    out = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(out.get() for _ in range(2))
    for rank, m, rate in res:
        assert m == 15.0                              # every rank reports the max over ranks
        assert abs(rate - 2 * 131072 * 10 / 0.015) < 1e-6 * rate


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
