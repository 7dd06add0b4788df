"""ts_tree_verify_attn_noalloc: the attention entry point for callers that
cannot allocate device memory (for example code whose device memory is all
owned by another runtime's allocator or a fixed budget).  It takes no
workspace and uses a static scratch array inside the library instead.

Checked through the C ABI, on two calls in a row with different shapes (the
second runs on scratch the first one left behind): against the ordinary
entry point (ts_tree_verify_attn with a caller-allocated workspace) and
against the fp64 oracle, with the device status read through
ts_noalloc_status after each call.  Then the array is left as a failed call
could leave it -- a timeout in its status word and non-zero hand-off
tickets (ts_noalloc_selftest) -- and the next calls must still be right,
with the status kept until the caller clears it.  This file is collected
last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import lossless_ultra_long_b200 as L
from lossless_ultra_long_b200 import inputs as I
from helpers import dev_bf16, sample_rows

pytestmark = pytest.mark.gpu

ATTN_TOL = 2e-3
SCRATCH_LIMIT = 7
TIMEOUT = 5


def _lib():
    lib = L.library()
    P = ctypes.c_void_p
    f = lib.ts_tree_verify_attn_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [P, P, P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int, P, ctypes.c_float, P, P]
    lib.ts_noalloc_status.restype = ctypes.c_int
    lib.ts_noalloc_status.argtypes = [P, ctypes.c_int]
    lib.ts_noalloc_selftest.restype = ctypes.c_int
    lib.ts_noalloc_selftest.argtypes = [P]
    return lib


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _call_noalloc(lib, q, k, v, n_ctx, parent, out):
    par = np.ascontiguousarray(parent, dtype=np.int32)
    t, hq, d = q.shape
    hkv, cap, _ = k.shape
    return lib.ts_tree_verify_attn_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), cap, hq, hkv, d, n_ctx, t,
        par.ctypes.data_as(ctypes.c_void_p), d ** -0.5, ctypes.c_void_p(out.data_ptr()), _stream())


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _check(lib, oracle_mod, w, count=24):
    """One no-alloc call: status 0, equal to the workspace entry point, and
    within 2e-3 of the oracle on sampled rows."""
    qh = I.gen_q(w)
    kh, vh = I.gen_kv(w)
    q, k, v = dev_bf16(qh), dev_bf16(kh), dev_bf16(vh)
    out = torch.full((w.n_tree, w.n_heads_q, w.head_dim), float("nan"), device="cuda")
    rc = _call_noalloc(lib, q, k, v, w.n_ctx, w.parent(), out)
    assert rc == 0, lib.ts_status_string(rc)
    ref = L.tree_verify_attn(q, k, v, w.n_ctx, w.parent())
    torch.cuda.synchronize()
    assert (out - ref).abs().max().item() <= ATTN_TOL, w.name
    nodes, heads = sample_rows(w.n_tree, w.n_heads_q, count, w.seed)
    want = oracle_mod.tree_verify_attn_rows(qh, kh, vh, w.n_ctx, w.parent(), nodes, heads)
    got = out.cpu().numpy().astype(np.float64)[nodes, heads]
    err = np.abs(got - want).max()
    assert err <= ATTN_TOL, f"{w.name}: {err}"


CASES = [I.LLAMA8B_32K, I.Workload("noalloc_b", 40, 8, 128, 7001, 13, seed=5)]


def test_noalloc_matches_workspace_entry_point_and_oracle_twice(oracle_mod):
    lib = _lib()
    for w in CASES:   # two calls in a row on the shared scratch
        _check(lib, oracle_mod, w)
        assert lib.ts_noalloc_status(_stream(), 0) == 0


def test_noalloc_status_survives_calls_until_cleared(oracle_mod):
    lib = _lib()
    assert lib.ts_noalloc_selftest(_stream()) == 0
    assert lib.ts_noalloc_status(_stream(), 0) == TIMEOUT   # read, not cleared
    # a call on the array as the failed call left it: still right, and the
    # earlier failure stays visible
    _check(lib, oracle_mod, CASES[1])
    assert lib.ts_noalloc_status(_stream(), 1) == TIMEOUT   # read and cleared
    assert lib.ts_noalloc_status(_stream(), 0) == 0
    _check(lib, oracle_mod, CASES[0])
    assert lib.ts_noalloc_status(_stream(), 0) == 0


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = _lib()
    hq, hkv, d, n_ctx, t = 1024, 8, 128, 4096, 64
    need = L.tree_verify_attn_workspace_size(hq, hkv, d, n_ctx, t)
    assert need > (16 << 20)
    dummy = ctypes.c_void_p(1 << 20)
    par = I.bfs_tree(t)
    rc = lib.ts_tree_verify_attn_noalloc(dummy, dummy, dummy, n_ctx + t, hq, hkv, d, n_ctx, t,
                                         par.ctypes.data_as(ctypes.c_void_p), 0.088, dummy, None)
    assert rc == SCRATCH_LIMIT


def test_noalloc_rejects_invalid_arguments_before_queueing_anything():
    lib = _lib()
    dummy = ctypes.c_void_p(1 << 20)
    par = I.bfs_tree(4)
    bad_par = np.array([-1, 0, 5, 1], np.int32)
    args = lambda p, hkv=2, scale=0.1: (dummy, dummy, dummy, 200, 8, hkv, 64, 100, 4,
                                        p.ctypes.data_as(ctypes.c_void_p), scale, dummy, None)
    assert lib.ts_tree_verify_attn_noalloc(*args(bad_par)) == 1
    assert lib.ts_tree_verify_attn_noalloc(*args(par, hkv=3)) == 1
    assert lib.ts_tree_verify_attn_noalloc(*args(par, scale=float("nan"))) == 1
    assert lib.ts_noalloc_status(None, 0) == 0
