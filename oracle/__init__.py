"""fp64 CPU oracle for the TokenSwift verification path (ctypes over ts_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, the smoke check and the
benchmark's CPU-baseline leg, never by the product library.  It shares no
code with the CUDA path; inputs come in as numpy arrays (bf16 as uint16 bit
patterns) from the seeded generators.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ts_oracle.c")
_LIB = os.path.join(_HERE, "libts_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ts_oracle.c with gcc (OpenMP, no fast-math) into libts_oracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        # a test that plants a mistake in the oracle loads its mutated build
        # from TSO_MUTANT_LIB (tests/test_oracle_mutants.py)
        lib = ctypes.CDLL(os.environ.get("TSO_MUTANT_LIB") or build())
        P = ctypes.c_void_p
        i32, i64, f64, f32 = ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_float
        lib.tso_tree_verify_attn.argtypes = [P, P, P, i64, i32, i32, i32, i32, i32, P, f64, P]
        lib.tso_tree_verify_attn_rows.argtypes = [P, P, P, i64, i32, i32, i32, i32, i32, P, f64,
                                                  P, P, i32, P]
        lib.tso_importance_scores.argtypes = [P, P, i64, i32, i32, i32, i32, f64, P]
        lib.tso_select_topk.argtypes = [P, i32, i32, i32, i32, P]
        lib.tso_gather_rows.argtypes = [P, i64, i32, i32, P, i32, P, i64]
        lib.tso_penalize_argmax.argtypes = [P, i32, i32, P, i32, f32, P, P]
        lib.tso_accept_longest.argtypes = [P, P, P, i32, P]
        lib.tso_penalize_argmax_path.argtypes = [P, i32, i32, P, i32, f32, P, P, P, P]
        lib.tso_accept_longest_random.argtypes = [P, P, P, i32, ctypes.c_uint64, P]
        lib.tso_sample_targets.argtypes = [P, P, i32, i32, f32, P]
        lib.tso_kv_commit_path.argtypes = [P, i64, i32, i32, i32, i32, P]
        _lib = lib
    return _lib


def set_num_threads(n: int) -> None:
    """Threads of the oracle's OpenMP loops from now on (in this process)."""
    _load()
    gomp = ctypes.CDLL("libgomp.so.1")
    gomp.omp_set_num_threads.argtypes = [ctypes.c_int]
    gomp.omp_set_num_threads(int(n))


def _p(a: np.ndarray):
    assert a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def tree_verify_attn(q, k, v, n_ctx: int, parent, scale: float | None = None) -> np.ndarray:
    """fp64 ``[T, Hq, D]``.  q: bf16 bits [T,Hq,D]; k, v: bf16 bits [Hkv, kv_cap, D]."""
    q, k, v, parent = _u16(q), _u16(k), _u16(v), _i32(parent)
    t, hq, d = q.shape
    hkv, cap, _ = k.shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    out = np.empty((t, hq, d), dtype=np.float64)
    rc = _load().tso_tree_verify_attn(_p(q), _p(k), _p(v), cap, hq, hkv, d, n_ctx, t, _p(parent),
                                      float(scale), _p(out))
    if rc != 0:
        raise ValueError("oracle: invalid attention arguments")
    return out


def tree_verify_attn_rows(q, k, v, n_ctx: int, parent, nodes, heads,
                          scale: float | None = None) -> np.ndarray:
    """fp64 ``[len(nodes), D]``: output rows (nodes[r], heads[r]) only."""
    q, k, v, parent = _u16(q), _u16(k), _u16(v), _i32(parent)
    nodes, heads = _i32(nodes), _i32(heads)
    t, hq, d = q.shape
    hkv, cap, _ = k.shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    out = np.empty((len(nodes), d), dtype=np.float64)
    rc = _load().tso_tree_verify_attn_rows(_p(q), _p(k), _p(v), cap, hq, hkv, d, n_ctx, t,
                                           _p(parent), float(scale), _p(nodes), _p(heads),
                                           len(nodes), _p(out))
    if rc != 0:
        raise ValueError("oracle: invalid attention arguments")
    return out


def importance_scores(q_last, k, n_ctx: int, n_heads_q: int, scale: float | None = None):
    """fp64 ``[Hkv, n_ctx]``.  q_last: bf16 bits [Hq, D]."""
    q_last, k = _u16(q_last), _u16(k)
    hkv, cap, d = k.shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    out = np.empty((hkv, n_ctx), dtype=np.float64)
    rc = _load().tso_importance_scores(_p(q_last), _p(k), cap, n_heads_q, hkv, d, n_ctx,
                                       float(scale), _p(out))
    if rc != 0:
        raise ValueError("oracle: invalid importance arguments")
    return out


def select_topk(scores, n_sink: int, budget: int) -> np.ndarray:
    """int32 ``[Hkv, n_keep]`` ascending.  scores: [Hkv, n_ctx], widened to fp64."""
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    hkv, n_ctx = scores.shape
    n_keep = min(n_ctx, n_sink + budget)
    idx = np.empty((hkv, max(n_keep, 0)), dtype=np.int32)
    rc = _load().tso_select_topk(_p(scores), hkv, n_ctx, n_sink, budget, _p(idx))
    if rc < 0:
        raise ValueError("oracle: invalid selection arguments")
    return idx


def gather_rows(src, idx, partial_cap: int | None = None) -> np.ndarray:
    src, idx = _u16(src), _i32(idx)
    hkv, cap, d = src.shape
    n_keep = idx.shape[1]
    pc = n_keep if partial_cap is None else partial_cap
    dst = np.zeros((hkv, pc, d), dtype=np.uint16)
    rc = _load().tso_gather_rows(_p(src), cap, hkv, d, _p(idx), n_keep, _p(dst), pc)
    if rc != 0:
        raise ValueError("oracle: invalid gather arguments")
    return dst


def penalize_argmax(logits, window, penalty: float = 1.2, return_penalized: bool = False):
    """int32 argmax ``[T]`` of the penalised fp32 logits (and optionally those logits)."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    window = _i32(window)
    t, vocab = logits.shape
    am = np.empty(t, dtype=np.int32)
    pen = np.empty_like(logits) if return_penalized else None
    rc = _load().tso_penalize_argmax(_p(logits), t, vocab, _p(window), len(window),
                                     float(np.float32(penalty)), _p(am),
                                     _p(pen) if pen is not None else None)
    if rc != 0:
        raise ValueError("oracle: invalid penalty arguments")
    return (am, pen) if return_penalized else am


def accept_longest(parent, tokens, argmax) -> np.ndarray:
    """int32 ``[2 + T]``: {len, bonus, path[0..len], unused...} (unused entries are -1)."""
    parent, tokens, argmax = _i32(parent), _i32(tokens), _i32(argmax)
    t = len(parent)
    out = np.full(2 + t, -1, dtype=np.int32)
    rc = _load().tso_accept_longest(_p(parent), _p(tokens), _p(argmax), t, _p(out))
    if rc < 0:
        raise ValueError("oracle: invalid tree")
    return out


def penalize_argmax_path(logits, window, parent, tokens, penalty: float = 1.2,
                         return_penalized: bool = False):
    """int32 argmax ``[T]`` with each node's draft-path tokens in its window."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    window, parent, tokens = _i32(window), _i32(parent), _i32(tokens)
    t, vocab = logits.shape
    am = np.empty(t, dtype=np.int32)
    pen = np.empty_like(logits) if return_penalized else None
    rc = _load().tso_penalize_argmax_path(_p(logits), t, vocab, _p(window), len(window),
                                          float(np.float32(penalty)), _p(parent), _p(tokens),
                                          _p(am), _p(pen) if pen is not None else None)
    if rc != 0:
        raise ValueError("oracle: invalid penalty arguments")
    return (am, pen) if return_penalized else am


def accept_longest_random(parent, tokens, argmax, r: int) -> np.ndarray:
    """As :func:`accept_longest`, the kept node being the (r mod c)-th of the
    c deepest valid nodes in index order."""
    parent, tokens, argmax = _i32(parent), _i32(tokens), _i32(argmax)
    t = len(parent)
    out = np.full(2 + t, -1, dtype=np.int32)
    rc = _load().tso_accept_longest_random(_p(parent), _p(tokens), _p(argmax), t,
                                           ctypes.c_uint64(int(r) & (2 ** 64 - 1)), _p(out))
    if rc < 0:
        raise ValueError("oracle: invalid tree")
    return out


def sample_targets(penalized, gumbel, temperature: float) -> np.ndarray:
    """int32 ``[T]``: per node the id maximising penalised / temperature + g
    (binary32), the Gumbel-max draw from softmax(penalised / temperature)."""
    penalized = np.ascontiguousarray(penalized, dtype=np.float32)
    gumbel = np.ascontiguousarray(gumbel, dtype=np.float32)
    if penalized.shape != gumbel.shape or penalized.ndim != 2:
        raise ValueError("oracle: penalised logits and noise must both be [T, V]")
    t, vocab = penalized.shape
    out = np.empty(t, dtype=np.int32)
    rc = _load().tso_sample_targets(_p(penalized), _p(gumbel), t, vocab,
                                    float(np.float32(temperature)), _p(out))
    if rc != 0:
        raise ValueError("oracle: invalid temperature")
    return out


def kv_commit_path(cache, n_ctx: int, n_tree: int, accept) -> np.ndarray:
    """A copy of one cache (bf16 bits [Hkv, kv_cap, D]) with the accepted
    path's tree rows moved to n_ctx + 0 .. n_ctx + L."""
    out = np.array(_u16(cache), copy=True)
    accept = _i32(accept)
    hkv, cap, d = out.shape
    rc = _load().tso_kv_commit_path(_p(out), cap, hkv, d, int(n_ctx), int(n_tree), _p(accept))
    if rc != 0:
        raise ValueError("oracle: invalid commit arguments")
    return out
