"""B200-native TokenSwift verification path: thin ctypes binding of libtsverify.so.

The three calls mirror the C ABI in ``include/ts_verify.h``; every step of
the path runs in the library's CUDA kernels.  This module only checks
tensor dtypes/devices, passes raw pointers and the current CUDA stream, and
turns non-zero status codes into exceptions.  torch supplies device memory
and streams.  There is no CPU fallback: if the library is not built, every
call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtsverify.so")

TS_MAX_TREE = 64
STATUS = {0: "TS_OK", 1: "TS_ERR_INVALID_ARG", 2: "TS_ERR_UNSUPPORTED", 3: "TS_ERR_WORKSPACE",
          4: "TS_ERR_CUDA", 5: "TS_ERR_TIMEOUT", 6: "TS_ERR_DEVICE_ARG"}

EXPORTS = ("ts_status_string", "ts_version", "ts_tree_verify_attn_workspace_size",
           "ts_tree_verify_attn", "ts_kv_importance_select_workspace_size",
           "ts_kv_importance_select", "ts_penalize_accept_workspace_size", "ts_penalize_accept",
           "ts_workspace_status", "ts_kernel_launch_count", "ts_tree_verify_attn_root_scores",
           "ts_kv_select_from_scores_workspace_size", "ts_kv_select_from_scores",
           "ts_ngram_table_bytes", "ts_ngram_init", "ts_ngram_update", "ts_ngram_topk",
           "ts_ngram_topk_prefix",
           "ts_ngram_count", "ts_ngram_size", "ts_selftest_bounded_wait",
           "ts_penalize_accept_ex", "ts_penalize_sample_accept", "ts_kv_commit_path")

TS_PENALIZE_PATH_TOKENS = 1
TS_ACCEPT_RANDOM_TIE = 2


class TsError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} "
                         f"({_lib().ts_status_string(status).decode()})")


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libtsverify.so is not built ({LIB_PATH}); run "
                               "`python -m lossless_ultra_long_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                                ctypes.c_size_t)
        lib.ts_status_string.restype = ctypes.c_char_p
        lib.ts_status_string.argtypes = [i32]
        lib.ts_version.restype = i32
        lib.ts_tree_verify_attn_workspace_size.restype = sz
        lib.ts_tree_verify_attn_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        lib.ts_tree_verify_attn.restype = i32
        lib.ts_tree_verify_attn.argtypes = [P, P, P, i64, i32, i32, i32, i32, i32, P, f32, P, P,
                                            sz, P]
        lib.ts_tree_verify_attn_root_scores.restype = i32
        lib.ts_tree_verify_attn_root_scores.argtypes = [P, P, P, i64, i32, i32, i32, i32, i32, P,
                                                        f32, P, P, P, sz, P]
        lib.ts_kv_select_from_scores_workspace_size.restype = sz
        lib.ts_kv_select_from_scores_workspace_size.argtypes = [i32, i32, i32]
        lib.ts_kv_select_from_scores.restype = i32
        lib.ts_kv_select_from_scores.argtypes = [P, P, P, i64, i32, i32, i32, i32, i32, i32, P, P,
                                                 P, P, i64, P, sz, P]
        lib.ts_kv_importance_select_workspace_size.restype = sz
        lib.ts_kv_importance_select_workspace_size.argtypes = [i32, i32, i32, i32]
        lib.ts_kv_importance_select.restype = i32
        lib.ts_kv_importance_select.argtypes = [P, P, P, i64, i32, i32, i32, i32, i32, i32, f32,
                                                P, P, P, P, i64, P, sz, P]
        lib.ts_penalize_accept_workspace_size.restype = sz
        lib.ts_penalize_accept_workspace_size.argtypes = [i32, i32]
        lib.ts_penalize_accept.restype = i32
        lib.ts_penalize_accept.argtypes = [P, i32, i32, P, i32, f32, P, P, P, P, P, sz, P]
        lib.ts_penalize_accept_ex.restype = i32
        lib.ts_penalize_accept_ex.argtypes = [P, i32, i32, P, i32, f32, P, P, ctypes.c_uint,
                                              ctypes.c_uint64, P, P, P, sz, P]
        lib.ts_penalize_sample_accept.restype = i32
        lib.ts_penalize_sample_accept.argtypes = [P, P, f32, i32, i32, P, i32, f32, P, P,
                                                  ctypes.c_uint, ctypes.c_uint64, P, P, P, sz, P]
        lib.ts_kv_commit_path.restype = i32
        lib.ts_kv_commit_path.argtypes = [P, P, i64, i32, i32, i32, i32, P, P, sz, P]
        lib.ts_kernel_launch_count.restype = ctypes.c_ulonglong
        lib.ts_kernel_launch_count.argtypes = []
        lib.ts_workspace_status.restype = i32
        lib.ts_workspace_status.argtypes = [P, P, i32]
        lib.ts_selftest_bounded_wait.restype = i32
        lib.ts_selftest_bounded_wait.argtypes = [P, sz, P]
        lib.ts_ngram_table_bytes.restype = sz
        lib.ts_ngram_table_bytes.argtypes = [i32, i64]
        lib.ts_ngram_init.restype = i32
        lib.ts_ngram_init.argtypes = [P, sz, i32, i64]
        lib.ts_ngram_update.restype = i32
        lib.ts_ngram_update.argtypes = [P, sz, P, i64, i64]
        lib.ts_ngram_topk.restype = i32
        lib.ts_ngram_topk.argtypes = [P, sz, ctypes.c_int32, i32, P, P, P]
        lib.ts_ngram_topk_prefix.restype = i32
        lib.ts_ngram_topk_prefix.argtypes = [P, sz, P, i32, i32, P, P, P]
        lib.ts_ngram_count.restype = i32
        lib.ts_ngram_count.argtypes = [P, sz, P, P]
        lib.ts_ngram_size.restype = i32
        lib.ts_ngram_size.argtypes = [P, sz, P, P]
        _LIB = lib
    return _LIB


def library():
    """The loaded ctypes handle (raises if the library is not built)."""
    return _lib()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check_dev(name, t, dtype, device=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the call's other tensors on {device}")


def _call_device(name, t):
    """The device a call runs on: that of its first tensor, which must be the
    current CUDA device (the kernels launch there, on its current stream)."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    cur = torch.cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"{name} is on {t.device} but the current device is cuda:{cur}")
    return t.device


def _ws_bytes(workspace, device):
    """Size in bytes of a workspace, after checking that it is a contiguous
    CUDA tensor on the call's device."""
    if not isinstance(workspace, torch.Tensor) or not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    if workspace.device != device:
        raise ValueError(f"workspace is on {workspace.device}, the call's tensors on {device}")
    if not workspace.is_contiguous():
        raise ValueError("workspace must be contiguous")
    return workspace.numel() * workspace.element_size()


def _host_i32(a):
    import numpy as np
    arr = np.ascontiguousarray(a.cpu().numpy() if isinstance(a, torch.Tensor) else a,
                               dtype=np.int32)
    return arr, arr.ctypes.data_as(ctypes.c_void_p)


def _raise(rc, where):
    if rc != 0:
        raise TsError(rc, where)


def new_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zero-filled uint8 device buffer (torch allocations are 512-byte aligned)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8,
                       device=device if device is not None else "cuda")


# ----------------------------------------------------------- attention
def tree_verify_attn_workspace_size(n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree) -> int:
    return int(_lib().ts_tree_verify_attn_workspace_size(n_heads_q, n_heads_kv, head_dim, n_ctx,
                                                         n_tree))


def tree_verify_attn(q, k_cache, v_cache, n_ctx: int, parent, out=None, workspace=None,
                     softmax_scale: float | None = None, stream=None, root_scores_out=None):
    """Tree-masked attention (``ts_tree_verify_attn``).

    q: bf16 [T, Hq, D]; k_cache, v_cache: bf16 [Hkv, kv_cap, D]; parent: host
    int32 [T].  Returns fp32 [T, Hq, D].  With ``root_scores_out`` (fp32
    [Hq, n_ctx]) it also leaves the root node's base-2 scores over the
    context (``ts_tree_verify_attn_root_scores``), the input of
    :func:`kv_select_from_scores`.
    """
    _check_dev("q", q, torch.bfloat16)
    dev = _call_device("q", q)
    _check_dev("k_cache", k_cache, torch.bfloat16, dev)
    _check_dev("v_cache", v_cache, torch.bfloat16, dev)
    t, hq, d = q.shape
    hkv, cap, d2 = k_cache.shape
    if v_cache.shape != k_cache.shape or d2 != d:
        raise ValueError("k_cache / v_cache / q shapes disagree")
    if out is None:
        out = torch.empty((t, hq, d), dtype=torch.float32, device=dev)
    _check_dev("out", out, torch.float32, dev)
    if workspace is None:
        workspace = new_workspace(tree_verify_attn_workspace_size(hq, hkv, d, n_ctx, t), dev)
    par, par_p = _host_i32(parent)
    if len(par) != t:
        raise ValueError("parent must have one entry per tree node")
    scale = float(d) ** -0.5 if softmax_scale is None else float(softmax_scale)
    ws_bytes = _ws_bytes(workspace, dev)
    if root_scores_out is None:
        rc = _lib().ts_tree_verify_attn(_ptr(q), _ptr(k_cache), _ptr(v_cache), cap, hq, hkv, d,
                                        int(n_ctx), t, par_p, scale, _ptr(out), _ptr(workspace),
                                        ws_bytes, _stream(stream))
        _raise(rc, "ts_tree_verify_attn")
        return out
    _check_dev("root_scores_out", root_scores_out, torch.float32, dev)
    if tuple(root_scores_out.shape) != (hq, int(n_ctx)):
        raise ValueError("root_scores_out must be [Hq, n_ctx]")
    rc = _lib().ts_tree_verify_attn_root_scores(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), cap, hq, hkv, d, int(n_ctx), t, par_p, scale,
        _ptr(out), _ptr(root_scores_out), _ptr(workspace), ws_bytes, _stream(stream))
    _raise(rc, "ts_tree_verify_attn_root_scores")
    return out


# ------------------------------------------------------------ selection
def kv_importance_select_workspace_size(n_heads_q, n_heads_kv, head_dim, n_ctx) -> int:
    return int(_lib().ts_kv_importance_select_workspace_size(n_heads_q, n_heads_kv, head_dim,
                                                             n_ctx))


def kv_importance_select(q_last, k_cache, v_cache, n_ctx: int, n_sink: int, budget: int,
                         k_partial=None, v_partial=None, idx_out=None, scores_out=None,
                         workspace=None, softmax_scale: float | None = None, stream=None,
                         want_scores: bool = False):
    """Sink + top-budget partial-KV update (``ts_kv_importance_select``).

    Returns ``(idx [Hkv, n_keep] int32, k_partial, v_partial, scores or None)``.
    """
    _check_dev("q_last", q_last, torch.bfloat16)
    dev = _call_device("q_last", q_last)
    _check_dev("k_cache", k_cache, torch.bfloat16, dev)
    _check_dev("v_cache", v_cache, torch.bfloat16, dev)
    hq, d = q_last.shape
    hkv, cap, d2 = k_cache.shape
    n_keep = min(n_ctx, n_sink + budget)
    if k_partial is None:
        k_partial = torch.empty((hkv, n_keep, d), dtype=torch.bfloat16, device=dev)
    if v_partial is None:
        v_partial = torch.empty_like(k_partial)
    if idx_out is None:
        idx_out = torch.empty((hkv, n_keep), dtype=torch.int32, device=dev)
    if want_scores and scores_out is None:
        scores_out = torch.empty((hkv, n_ctx), dtype=torch.float32, device=dev)
    for name, t, dt in (("k_partial", k_partial, torch.bfloat16),
                        ("v_partial", v_partial, torch.bfloat16),
                        ("idx_out", idx_out, torch.int32)):
        _check_dev(name, t, dt, dev)
    if scores_out is not None:
        _check_dev("scores_out", scores_out, torch.float32, dev)
    if workspace is None:
        workspace = new_workspace(kv_importance_select_workspace_size(hq, hkv, d, n_ctx), dev)
    scale = float(d) ** -0.5 if softmax_scale is None else float(softmax_scale)
    rc = _lib().ts_kv_importance_select(
        _ptr(q_last), _ptr(k_cache), _ptr(v_cache), cap, hq, hkv, d, int(n_ctx), int(n_sink),
        int(budget), scale, _ptr(scores_out), _ptr(idx_out), _ptr(k_partial), _ptr(v_partial),
        k_partial.shape[1], _ptr(workspace), _ws_bytes(workspace, dev), _stream(stream))
    _raise(rc, "ts_kv_importance_select")
    return idx_out, k_partial, v_partial, scores_out


def kv_select_from_scores_workspace_size(n_heads_q, n_heads_kv, n_ctx) -> int:
    return int(_lib().ts_kv_select_from_scores_workspace_size(n_heads_q, n_heads_kv, n_ctx))


def kv_select_from_scores(root_scores, k_cache, v_cache, n_ctx: int, n_sink: int, budget: int,
                          k_partial=None, v_partial=None, idx_out=None, scores_out=None,
                          workspace=None, stream=None, want_scores: bool = False):
    """The partial-KV update from root scores left by the verify attention
    (``ts_kv_select_from_scores``).  root_scores: fp32 [Hq, n_ctx] (base 2).

    Returns ``(idx [Hkv, n_keep] int32, k_partial, v_partial, scores or None)``.
    """
    _check_dev("root_scores", root_scores, torch.float32)
    dev = _call_device("root_scores", root_scores)
    _check_dev("k_cache", k_cache, torch.bfloat16, dev)
    _check_dev("v_cache", v_cache, torch.bfloat16, dev)
    hq, n = root_scores.shape
    if n != int(n_ctx):
        raise ValueError("root_scores must be [Hq, n_ctx]")
    hkv, cap, d = k_cache.shape
    n_keep = min(n_ctx, n_sink + budget)
    if k_partial is None:
        k_partial = torch.empty((hkv, n_keep, d), dtype=torch.bfloat16, device=dev)
    if v_partial is None:
        v_partial = torch.empty_like(k_partial)
    if idx_out is None:
        idx_out = torch.empty((hkv, n_keep), dtype=torch.int32, device=dev)
    if want_scores and scores_out is None:
        scores_out = torch.empty((hkv, n_ctx), dtype=torch.float32, device=dev)
    for name, t, dt in (("k_partial", k_partial, torch.bfloat16),
                        ("v_partial", v_partial, torch.bfloat16),
                        ("idx_out", idx_out, torch.int32)):
        _check_dev(name, t, dt, dev)
    if scores_out is not None:
        _check_dev("scores_out", scores_out, torch.float32, dev)
    if workspace is None:
        workspace = new_workspace(kv_select_from_scores_workspace_size(hq, hkv, int(n_ctx)), dev)
    rc = _lib().ts_kv_select_from_scores(
        _ptr(root_scores), _ptr(k_cache), _ptr(v_cache), cap, hq, hkv, d, int(n_ctx),
        int(n_sink), int(budget), _ptr(scores_out), _ptr(idx_out), _ptr(k_partial),
        _ptr(v_partial), k_partial.shape[1], _ptr(workspace), _ws_bytes(workspace, dev),
        _stream(stream))
    _raise(rc, "ts_kv_select_from_scores")
    return idx_out, k_partial, v_partial, scores_out


# ------------------------------------------------------ penalty + accept
def penalize_accept_workspace_size(n_tree, vocab) -> int:
    return int(_lib().ts_penalize_accept_workspace_size(n_tree, vocab))


def penalize_accept(logits, window, penalty: float, parent, tree_tokens, argmax_out=None,
                    accept_out=None, workspace=None, stream=None, want_argmax: bool = True,
                    flags: int = 0, random: int = 0):
    """Contextual penalty + per-node argmax + longest accepted path
    (``ts_penalize_accept``; with ``flags`` -- TS_PENALIZE_PATH_TOKENS,
    TS_ACCEPT_RANDOM_TIE -- ``ts_penalize_accept_ex``, ``random`` the
    caller's random 64-bit integer for the choice among the deepest valid
    nodes).

    Returns ``(accept [2 + T] int32, argmax [T] int32 or None)``.
    """
    _check_dev("logits", logits, torch.float32)
    dev = _call_device("logits", logits)
    _check_dev("tree_tokens", tree_tokens, torch.int32, dev)
    t, vocab = logits.shape
    if window is not None and window.numel() > 0:
        _check_dev("window", window, torch.int32, dev)
        wlen, wptr = window.numel(), _ptr(window)
    else:
        wlen, wptr = 0, None
    if accept_out is None:
        accept_out = torch.empty(2 + t, dtype=torch.int32, device=dev)
    if want_argmax and argmax_out is None:
        argmax_out = torch.empty(t, dtype=torch.int32, device=dev)
    _check_dev("accept_out", accept_out, torch.int32, dev)
    if argmax_out is not None:
        _check_dev("argmax_out", argmax_out, torch.int32, dev)
    if workspace is None:
        workspace = new_workspace(penalize_accept_workspace_size(t, vocab), dev)
    par, par_p = _host_i32(parent)
    if len(par) != t:
        raise ValueError("parent must have one entry per tree node")
    if flags == 0:
        rc = _lib().ts_penalize_accept(_ptr(logits), t, vocab, wptr, wlen, float(penalty), par_p,
                                       _ptr(tree_tokens), _ptr(argmax_out), _ptr(accept_out),
                                       _ptr(workspace), _ws_bytes(workspace, dev),
                                       _stream(stream))
        _raise(rc, "ts_penalize_accept")
    else:
        rc = _lib().ts_penalize_accept_ex(
            _ptr(logits), t, vocab, wptr, wlen, float(penalty), par_p, _ptr(tree_tokens),
            int(flags), int(random) & (2 ** 64 - 1), _ptr(argmax_out), _ptr(accept_out),
            _ptr(workspace), _ws_bytes(workspace, dev), _stream(stream))
        _raise(rc, "ts_penalize_accept_ex")
    return accept_out, argmax_out


def penalize_sample_accept(logits, gumbel, temperature: float, window, penalty: float, parent,
                           tree_tokens, target_out=None, accept_out=None, workspace=None,
                           stream=None, want_target: bool = True, flags: int = 0,
                           random: int = 0):
    """Contextual penalty + per-node temperature draw + longest accepted path
    (``ts_penalize_sample_accept``): node i's target token is the id
    maximising penalised / temperature + gumbel[i] (binary32), the
    Gumbel-max draw from softmax(penalised / temperature); ``gumbel`` is the
    caller's standard Gumbel noise, fp32 ``[T, V]`` on the device.  ``flags``
    and ``random`` as for :func:`penalize_accept`.

    Returns ``(accept [2 + T] int32, target [T] int32 or None)``.
    """
    _check_dev("logits", logits, torch.float32)
    dev = _call_device("logits", logits)
    _check_dev("gumbel", gumbel, torch.float32, dev)
    _check_dev("tree_tokens", tree_tokens, torch.int32, dev)
    t, vocab = logits.shape
    if tuple(gumbel.shape) != (t, vocab):
        raise ValueError("gumbel must have the logits' shape [T, V]")
    if window is not None and window.numel() > 0:
        _check_dev("window", window, torch.int32, dev)
        wlen, wptr = window.numel(), _ptr(window)
    else:
        wlen, wptr = 0, None
    if accept_out is None:
        accept_out = torch.empty(2 + t, dtype=torch.int32, device=dev)
    if want_target and target_out is None:
        target_out = torch.empty(t, dtype=torch.int32, device=dev)
    _check_dev("accept_out", accept_out, torch.int32, dev)
    if target_out is not None:
        _check_dev("target_out", target_out, torch.int32, dev)
    if workspace is None:
        workspace = new_workspace(penalize_accept_workspace_size(t, vocab), dev)
    par, par_p = _host_i32(parent)
    if len(par) != t:
        raise ValueError("parent must have one entry per tree node")
    rc = _lib().ts_penalize_sample_accept(
        _ptr(logits), _ptr(gumbel), float(temperature), t, vocab, wptr, wlen, float(penalty),
        par_p, _ptr(tree_tokens), int(flags), int(random) & (2 ** 64 - 1), _ptr(target_out),
        _ptr(accept_out), _ptr(workspace), _ws_bytes(workspace, dev), _stream(stream))
    _raise(rc, "ts_penalize_sample_accept")
    return accept_out, target_out


def kv_commit_path(k_cache, v_cache, n_ctx: int, n_tree: int, accept, workspace=None,
                   stream=None):
    """Moves the accepted path's tree rows to n_ctx + 0 .. n_ctx + L in both
    caches, in place (``ts_kv_commit_path``); ``accept`` is the device
    result of :func:`penalize_accept`."""
    _check_dev("k_cache", k_cache, torch.bfloat16)
    dev = _call_device("k_cache", k_cache)
    _check_dev("v_cache", v_cache, torch.bfloat16, dev)
    _check_dev("accept", accept, torch.int32, dev)
    hkv, cap, d = k_cache.shape
    if v_cache.shape != k_cache.shape:
        raise ValueError("k_cache / v_cache shapes disagree")
    if workspace is None:
        workspace = new_workspace(256, dev)
    rc = _lib().ts_kv_commit_path(_ptr(k_cache), _ptr(v_cache), cap, hkv, d, int(n_ctx),
                                  int(n_tree), _ptr(accept), _ptr(workspace),
                                  _ws_bytes(workspace, dev), _stream(stream))
    _raise(rc, "ts_kv_commit_path")
    return k_cache, v_cache


def kernel_launch_count() -> int:
    """Kernels the library has launched in this process."""
    return int(_lib().ts_kernel_launch_count())


def selftest_bounded_wait(workspace=None, stream=None):
    """``ts_selftest_bounded_wait``: one CTA takes the kernels' bounded wait
    on a barrier nothing completes; about a second later TS_ERR_TIMEOUT is
    in the workspace's status word.  Returns the workspace."""
    if workspace is None:
        workspace = new_workspace(256)
    nbytes = _ws_bytes(workspace, _call_device("workspace", workspace))
    _raise(_lib().ts_selftest_bounded_wait(_ptr(workspace), nbytes, _stream(stream)),
           "ts_selftest_bounded_wait")
    return workspace


def workspace_status(workspace, clear: bool = True, stream=None) -> int:
    """Device-side status word of a workspace (synchronises the stream)."""
    _ws_bytes(workspace, _call_device("workspace", workspace))
    return int(_lib().ts_workspace_status(_ptr(workspace), _stream(stream), int(clear)))


# --------------------------------------------------------- n-gram reuse table
class NgramTable:
    """The n-gram reuse table (``ts_ngram_*``) in a host buffer this object
    owns.  ``update(text, n_new)`` counts the n-grams of ``text`` that end
    at its last ``n_new`` tokens; ``topk(first, k)`` returns the most
    frequent ones starting with ``first`` as ``(continuations [m, n-1],
    counts [m])``, count descending, ties by continuation ascending;
    ``topk_prefix(prefix, k)`` does the same for a prefix of 1 to n-1
    tokens (n-1 tokens: the next-token counts)."""

    def __init__(self, n: int, capacity: int):
        import numpy as np
        nbytes = int(_lib().ts_ngram_table_bytes(int(n), int(capacity)))
        if nbytes == 0:
            raise ValueError("n must be in [2, 8] and capacity a power of two >= 2")
        self.n, self.capacity, self.nbytes = int(n), int(capacity), nbytes
        self._buf = np.empty((nbytes + 7) // 8, dtype=np.uint64)   # 8-byte aligned
        self._p = self._buf.ctypes.data_as(ctypes.c_void_p)
        _raise(_lib().ts_ngram_init(self._p, nbytes, self.n, self.capacity), "ts_ngram_init")

    def update(self, text, n_new: int | None = None) -> None:
        arr, p = _host_i32(text)
        n_new = len(arr) if n_new is None else int(n_new)
        _raise(_lib().ts_ngram_update(self._p, self.nbytes, p, len(arr), n_new),
               "ts_ngram_update")

    def topk(self, first: int, k: int):
        import numpy as np
        cont = np.empty((int(k), self.n - 1), dtype=np.int32)
        cnt = np.empty(int(k), dtype=np.int64)
        found = ctypes.c_int(0)
        _raise(_lib().ts_ngram_topk(self._p, self.nbytes, int(first), int(k),
                                    cont.ctypes.data_as(ctypes.c_void_p),
                                    cnt.ctypes.data_as(ctypes.c_void_p), ctypes.byref(found)),
               "ts_ngram_topk")
        return cont[:found.value], cnt[:found.value]

    def topk_prefix(self, prefix, k: int):
        """The k most frequent n-grams that start with ``prefix`` (1 to n-1
        tokens): ``(continuations [m, n - len(prefix)], counts [m])``."""
        import numpy as np
        arr, p = _host_i32(prefix)
        cont = np.empty((int(k), max(self.n - len(arr), 0)), dtype=np.int32)
        cnt = np.empty(int(k), dtype=np.int64)
        found = ctypes.c_int(0)
        _raise(_lib().ts_ngram_topk_prefix(self._p, self.nbytes, p, len(arr), int(k),
                                           cont.ctypes.data_as(ctypes.c_void_p),
                                           cnt.ctypes.data_as(ctypes.c_void_p),
                                           ctypes.byref(found)),
               "ts_ngram_topk_prefix")
        return cont[:found.value], cnt[:found.value]

    def count(self, gram) -> int:
        arr, p = _host_i32(gram)
        if len(arr) != self.n:
            raise ValueError(f"an n-gram has {self.n} tokens")
        c = ctypes.c_int64(0)
        _raise(_lib().ts_ngram_count(self._p, self.nbytes, p, ctypes.byref(c)), "ts_ngram_count")
        return int(c.value)

    def size(self):
        """(distinct n-grams held, n-grams counted)."""
        d, t = ctypes.c_int64(0), ctypes.c_int64(0)
        _raise(_lib().ts_ngram_size(self._p, self.nbytes, ctypes.byref(d), ctypes.byref(t)),
               "ts_ngram_size")
        return int(d.value), int(t.value)
