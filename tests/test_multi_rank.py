"""bench.py's multi-process path on CPU (gloo, world size 2).

The path shards as independent replicas (one per GPU, no data-path
collective): the host logic that N > 1 adds is the environment parsing, the
max over ranks of every device time, the whole-job value (work of all ranks
over the slowest rank's time) and the rank-0-only output of the reference
arm.  Those run here as two gloo processes; the GPU path calls the same
functions over NCCL.
"""
import os
import socket
import subprocess
import sys
from datetime import timedelta

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        ms = bench.max_over_ranks([10.0 + rank, 5.0 * (world - rank)])
        val = bench.job_tflops(2.0e12, world, ms[0])
        q.put((rank, ms, val, bench.init_dist(None)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_world2():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        results = sorted(q.get(timeout=120) for _ in range(2))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.terminate()
    assert [p.exitcode for p in procs] == [0, 0]
    for rank, ms, val, env in results:
        assert ms == [11.0, 10.0]                     # the slowest rank's time, element-wise
        assert val == pytest.approx(2.0e12 * 2 / 11.0e-3 / 1e12)
        assert env == (2, rank, rank)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.5]) == [3.0, 4.5]
    assert bench.job_tflops(1e12, 1, 1.0) == pytest.approx(1000.0)  # 1e12 flops in 1 ms


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "5", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
