"""The bench's multi-rank logic on CPU with world_size-2 gloo process groups (no GPU).

With N GPUs every rank times its own batch; the reported step time is the slowest
rank's (max over ranks) and the value is the whole job's throughput.  The reference
arm runs on rank 0 only.
"""

import datetime
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        step_ms = [2.0, 3.0][rank]          # rank 1 is the slow one
        kernels = [1.5 - rank, 0.5 + rank]  # each rank slowest on a different kernel
        a = bench.max_over_ranks([step_ms] + kernels, device="cpu")
        b = bench.max_over_ranks([10.0 * (rank + 1)], device="cpu")
        v = bench.whole_job_tflops(world, 68.72e9, a[0])
        dist.barrier()
        q.put((rank, a, b, v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_with_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, a, b, v in res:
        assert a == [3.0, 1.5, 1.5], (rank, a)  # every value is the slowest rank's
        assert b == [20.0]
        assert abs(v - 2 * 68.72e9 / 3e-3 / 1e12) < 1e-9  # both ranks' work over the slowest time


def test_max_over_ranks_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.0, 2.5]) == [1.0, 2.5]
    assert bench.whole_job_tflops(1, 1e12, 1000.0) == 1.0


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the non-zero ranks of `--impl reference` exit 0 at once, printing nothing."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
