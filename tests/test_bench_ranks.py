"""The multi-rank path of bench.py, on the CPU: world size 2 over gloo.

bench.py --gpus N runs N independent replicas of the step (the path has no
data-path exchange); the only cross-rank work is taking the slowest rank's
duration, and the job's throughput counts every rank's steps.  The
reference arm prints from rank 0 only; other ranks return without work.
"""
import argparse
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        sys.path.insert(0, ROOT)
        import bench as b
        ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
        m = b.max_over_ranks(ms, world, "cpu")
        v = b.job_throughput(100, world, m)
        dist.barrier()
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0]
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, m, v in got:
        assert m == 15.0                       # both ranks see the slowest
        assert v == pytest.approx(2 * 100 / 0.015)


def test_single_process_reduction_is_identity():
    assert bench.max_over_ranks(12.5, 1, "cpu") == 12.5
    assert bench.job_throughput(1000, 1, 250.0) == pytest.approx(4000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(steps=3, warmup=1, gpus=2, impl="reference")
    assert bench.run_reference(args) is None


def test_ngram_host_timing_runs_on_the_cpu():
    from lossless_ultra_long_b200 import build
    build.build()
    import lossless_ultra_long_b200 as L
    us = bench.ngram_host_timing(L, n_tokens=3000, steps=50)
    assert 0.0 < us < 1e5
