"""ts_tree_verify_attn_noalloc: the attention entry point for callers that
cannot allocate device memory (for example code whose device memory is all
owned by another runtime's allocator or a fixed budget).  It takes no
workspace and uses a static scratch array inside the library instead.

Checked through the C ABI against the ordinary entry point
(ts_tree_verify_attn with a caller-allocated workspace), on two calls in a
row with different shapes, so the second call runs on scratch the first one
left behind.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import lossless_ultra_long_b200 as L
from lossless_ultra_long_b200 import inputs as I
from helpers import dev_bf16

pytestmark = pytest.mark.gpu

ATTN_TOL = 2e-3
SCRATCH_LIMIT = 7


def _noalloc_fn():
    lib = L.library()
    f = lib.ts_tree_verify_attn_noalloc
    P = ctypes.c_void_p
    f.restype = ctypes.c_int
    f.argtypes = [P, P, P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int, P, ctypes.c_float, P, P]
    return f


def _call_noalloc(f, q, k, v, n_ctx, parent, out):
    par = np.ascontiguousarray(parent, dtype=np.int32)
    t, hq, d = q.shape
    hkv, cap, _ = k.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return f(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
             ctypes.c_void_p(v.data_ptr()), cap, hq, hkv, d, n_ctx, t,
             par.ctypes.data_as(ctypes.c_void_p), d ** -0.5, ctypes.c_void_p(out.data_ptr()),
             stream)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_noalloc_matches_workspace_entry_point_twice():
    f = _noalloc_fn()
    cases = [I.LLAMA8B_32K, I.Workload("noalloc_b", 40, 8, 128, 7001, 13, seed=5)]
    for w in cases:   # two calls in a row on the shared scratch
        q = dev_bf16(I.gen_q(w))
        k, v = (dev_bf16(x) for x in I.gen_kv(w))
        out = torch.full((w.n_tree, w.n_heads_q, w.head_dim), float("nan"), device="cuda")
        rc = _call_noalloc(f, q, k, v, w.n_ctx, w.parent(), out)
        assert rc == 0, L.library().ts_status_string(rc)
        ref = L.tree_verify_attn(q, k, v, w.n_ctx, w.parent())
        torch.cuda.synchronize()
        err = (out - ref).abs().max().item()
        assert err <= ATTN_TOL, f"{w.name}: {err}"


def test_noalloc_rejects_problems_beyond_its_scratch():
    f = _noalloc_fn()
    hq, hkv, d, n_ctx, t = 1024, 8, 128, 4096, 64
    need = L.tree_verify_attn_workspace_size(hq, hkv, d, n_ctx, t)
    assert need > (16 << 20)
    dummy = ctypes.c_void_p(1 << 20)
    par = I.bfs_tree(t)
    rc = f(dummy, dummy, dummy, n_ctx + t, hq, hkv, d, n_ctx, t,
           par.ctypes.data_as(ctypes.c_void_p), 0.088, dummy, None)
    assert rc == SCRATCH_LIMIT
