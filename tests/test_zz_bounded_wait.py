"""Failure detection without a GPU fault.

On the GPU: the kernels' bounded wait is made to run out on a barrier that
nothing completes (ts_selftest_bounded_wait); the timeout is read from the
workspace status word on the host and the same context then runs the path
correctly.  Nothing traps, faults or spins without limit.

On the CPU (gloo, two ranks): a rank that dies before the bench's one
cross-rank step (the max over ranks) makes the other rank's collective end
with an error within the process group's timeout instead of waiting for
good.
"""
import datetime
import os
import socket
import sys
import time

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_bounded_wait_runs_out_and_the_context_stays_usable(oracle_mod):
    import torch
    import lossless_ultra_long_b200 as L
    from lossless_ultra_long_b200 import inputs as I
    from helpers import dev_bf16
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    t0 = time.perf_counter()
    ws = L.selftest_bounded_wait()
    assert L.workspace_status(ws) == 5          # TS_ERR_TIMEOUT, read on the host
    waited = time.perf_counter() - t0
    assert 0.2 < waited < 30.0, waited          # about one second of SM clock
    assert L.workspace_status(ws) == 0          # cleared by the read
    # the context still works: one small verification call against the oracle
    w = I.TINY
    q = I.gen_q(w)
    k, v = I.gen_kv(w)
    out = L.tree_verify_attn(dev_bf16(q), dev_bf16(k), dev_bf16(v), w.n_ctx, w.parent())
    torch.cuda.synchronize()
    want = oracle_mod.tree_verify_attn(q, k, v, w.n_ctx, w.parent())
    assert np.abs(out.cpu().numpy() - want).max() <= 2e-3


def test_selftest_rejects_a_missing_workspace_on_the_host():
    import ctypes
    from lossless_ultra_long_b200 import build
    build.build()
    import lossless_ultra_long_b200 as L
    lib = L.library()
    assert lib.ts_selftest_bounded_wait(None, 256, None) == 3
    assert lib.ts_selftest_bounded_wait(ctypes.c_void_p(1 << 20), 64, None) == 3


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=10))
    if rank == 1:
        os._exit(3)                              # dies before the collective
    sys.path.insert(0, ROOT)
    import bench
    t0 = time.time()
    try:
        bench.max_over_ranks(1.0, world, "cpu")
        q.put(("returned", time.time() - t0))
    except Exception as e:                       # the failure reaches this rank
        q.put((type(e).__name__, time.time() - t0))
    os._exit(0)


def test_a_dead_rank_ends_the_others_collective_with_an_error():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    alive = [p.is_alive() for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert alive == [False, False]
    assert [p.exitcode for p in procs] == [0, 3]
    what, took = q.get(timeout=5)
    assert what != "returned", "the collective completed without the dead rank"
    assert took < 60.0
