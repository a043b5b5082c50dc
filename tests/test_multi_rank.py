"""Replica plumbing of bench.py with two gloo ranks on CPU.

The decode step shards by request with no exchange, so multi-GPU runs are
independent replicas; what needs checking is the host side around them: the
barrier, the max of the ranks' device times, the whole-job aggregate, and
that the reference arm prints from rank 0 only.
"""
import os
import socket
import subprocess
import sys
from pathlib import Path

import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, str(ROOT))
    import bench
    reps = bench.Replicas("gloo")
    reps.barrier()
    local_ms = [1.25, 2.0][rank]  # rank 1 is the slow one
    worst = reps.max_over_ranks(local_ms)
    gbs = bench.whole_job_gbs(reps.world, 10**9, worst)
    reps.barrier()
    reps.close()
    q.put((rank, worst, gbs))


def test_two_gloo_ranks_time_the_job_by_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, worst, gbs in res:
        assert worst == 2.0                      # max over ranks, on every rank
        assert abs(gbs - 2 * 1.0 / 2.0e-3) < 1e-9  # 2 replicas x 1 GB per 2 ms


def test_reference_arm_prints_on_rank_zero_only():
    """Under torchrun every rank runs bench.py --impl reference; rank 0 alone works."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--steps", "1", "--warmup", "3"], env=env,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""
