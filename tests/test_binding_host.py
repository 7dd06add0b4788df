"""The Python binding's marshalling, on a machine without a GPU.

Host tensors wrapped in a subclass that reports a CUDA device stand in for
device tensors, so every entry point's argument checks and marshalling run
here: with valid arguments the library's own host checks accept the call,
which then ends at its first CUDA runtime call with TS_ERR_CUDA (there is no
device to launch on); tensors on another device, a host workspace or a
non-current device are refused by the binding before the library is called.

Skipped wherever a GPU is present: there these host pointers would reach
real kernels.
"""
import types

import numpy as np
import pytest
import torch

import lossless_ultra_long_b200 as L
from lossless_ultra_long_b200 import inputs as I

pytestmark = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="host-memory stand-ins are for machines without a GPU")

TS_ERR_CUDA = 4
STREAM = types.SimpleNamespace(cuda_stream=0)
T, HQ, HKV, D, N_CTX, VOCAB = 13, 8, 2, 64, 2048, 4096


class _OnDevice(torch.Tensor):
    """A host tensor that reports itself as living on cuda:<_index>."""

    @property
    def is_cuda(self):
        return True

    @property
    def device(self):
        return torch.device("cuda", getattr(self, "_index", 0))


def on_dev(t, index=0):
    f = torch.Tensor._make_subclass(_OnDevice, t.contiguous())
    f._index = index
    return f


def zeros(shape, dtype=torch.float32, index=0):
    return on_dev(torch.zeros(shape, dtype=dtype), index)


def workspace(n=1 << 24, index=0):
    buf = torch.zeros(n + 256, dtype=torch.uint8)
    off = (-buf.data_ptr()) % 256   # the library wants 256-byte aligned workspaces
    return on_dev(buf[off:off + n], index)


@pytest.fixture(autouse=True)
def _current_device_zero(monkeypatch):
    L.library()
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)


def _attn_inputs(index=0):
    q = zeros((T, HQ, D), torch.bfloat16, index)
    k = zeros((HKV, N_CTX + T, D), torch.bfloat16)
    v = zeros((HKV, N_CTX + T, D), torch.bfloat16)
    return q, k, v


def _partials():
    return dict(k_partial=zeros((HKV, 256, D), torch.bfloat16),
                v_partial=zeros((HKV, 256, D), torch.bfloat16),
                idx_out=zeros((HKV, 256), torch.int32))


CALLS = {
    "tree_verify_attn": lambda: L.tree_verify_attn(
        *_attn_inputs(), N_CTX, I.bfs_tree(T), out=zeros((T, HQ, D)), workspace=workspace(),
        stream=STREAM),
    "tree_verify_attn_root_scores": lambda: L.tree_verify_attn(
        *_attn_inputs(), N_CTX, I.bfs_tree(T), out=zeros((T, HQ, D)), workspace=workspace(),
        root_scores_out=zeros((HQ, N_CTX)), stream=STREAM),
    "kv_importance_select": lambda: L.kv_importance_select(
        zeros((HQ, D), torch.bfloat16), *_attn_inputs()[1:], N_CTX, 16, 240, **_partials(),
        workspace=workspace(), stream=STREAM),
    "kv_select_from_scores": lambda: L.kv_select_from_scores(
        zeros((HQ, N_CTX)), *_attn_inputs()[1:], N_CTX, 16, 240, **_partials(),
        workspace=workspace(), stream=STREAM),
    "penalize_accept": lambda: L.penalize_accept(
        zeros((T, VOCAB)), zeros(16, torch.int32), 1.2, I.bfs_tree(T), zeros(T, torch.int32),
        argmax_out=zeros(T, torch.int32), accept_out=zeros(2 + T, torch.int32),
        workspace=workspace(), stream=STREAM),
    "penalize_accept_ex": lambda: L.penalize_accept(
        zeros((T, VOCAB)), zeros(16, torch.int32), 1.2, I.bfs_tree(T), zeros(T, torch.int32),
        argmax_out=zeros(T, torch.int32), accept_out=zeros(2 + T, torch.int32),
        workspace=workspace(), stream=STREAM,
        flags=L.TS_PENALIZE_PATH_TOKENS | L.TS_ACCEPT_RANDOM_TIE, random=5),
    "penalize_sample_accept": lambda: L.penalize_sample_accept(
        zeros((T, VOCAB)), zeros((T, VOCAB)), 0.7, zeros(16, torch.int32), 1.2, I.bfs_tree(T),
        zeros(T, torch.int32), target_out=zeros(T, torch.int32),
        accept_out=zeros(2 + T, torch.int32), workspace=workspace(), stream=STREAM),
    "kv_commit_path": lambda: L.kv_commit_path(
        *_attn_inputs()[1:], N_CTX, T, zeros(2 + T, torch.int32), workspace=workspace(),
        stream=STREAM),
    "selftest_bounded_wait": lambda: L.selftest_bounded_wait(workspace=workspace(),
                                                             stream=STREAM),
}


@pytest.mark.parametrize("name", sorted(CALLS))
def test_valid_call_passes_every_host_check(name):
    with pytest.raises(L.TsError) as e:
        CALLS[name]()
    assert e.value.status == TS_ERR_CUDA, name


def test_workspace_status_reaches_the_runtime():
    assert L.workspace_status(workspace(), stream=STREAM) == TS_ERR_CUDA


def test_tensors_on_another_device_are_refused():
    q, k, v = _attn_inputs()
    with pytest.raises(ValueError, match="k_cache is on cuda:1"):
        L.tree_verify_attn(q, zeros(k.shape, torch.bfloat16, 1), v, N_CTX, I.bfs_tree(T),
                           out=zeros((T, HQ, D)), workspace=workspace(), stream=STREAM)
    with pytest.raises(ValueError, match="window is on cuda:1"):
        L.penalize_accept(zeros((T, VOCAB)), zeros(16, torch.int32, 1), 1.2, I.bfs_tree(T),
                          zeros(T, torch.int32), workspace=workspace(),
                          argmax_out=zeros(T, torch.int32), accept_out=zeros(2 + T, torch.int32),
                          stream=STREAM)
    with pytest.raises(ValueError, match="gumbel is on cuda:1"):
        L.penalize_sample_accept(zeros((T, VOCAB)), zeros((T, VOCAB), index=1), 0.7, None, 1.2,
                                 I.bfs_tree(T), zeros(T, torch.int32),
                                 target_out=zeros(T, torch.int32),
                                 accept_out=zeros(2 + T, torch.int32), workspace=workspace(),
                                 stream=STREAM)
    with pytest.raises(ValueError, match="workspace is on cuda:1"):
        L.kv_commit_path(k, v, N_CTX, T, zeros(2 + T, torch.int32), workspace=workspace(index=1),
                         stream=STREAM)


def test_a_call_off_the_current_device_is_refused():
    q, k, v = (on_dev(t, 1) for t in _attn_inputs())
    with pytest.raises(ValueError, match="current device is cuda:0"):
        L.tree_verify_attn(q, k, v, N_CTX, I.bfs_tree(T), out=zeros((T, HQ, D), index=1),
                           workspace=workspace(index=1), stream=STREAM)


def test_host_or_strided_workspaces_are_refused():
    q, k, v = _attn_inputs()
    for ws, msg in ((torch.zeros(1 << 20, dtype=torch.uint8), "must be a CUDA tensor"),
                    (on_dev(torch.zeros((2, 1 << 20), dtype=torch.uint8)).t(), "contiguous")):
        with pytest.raises(ValueError, match=msg):
            L.tree_verify_attn(q, k, v, N_CTX, I.bfs_tree(T), out=zeros((T, HQ, D)),
                               workspace=ws, stream=STREAM)


def test_host_checks_of_the_library_still_apply():
    """A call the library rejects on the host never reaches the runtime."""
    with pytest.raises(L.TsError) as e:
        L.penalize_sample_accept(zeros((T, VOCAB)), zeros((T, VOCAB)), float("nan"), None, 1.2,
                                 I.bfs_tree(T), zeros(T, torch.int32),
                                 target_out=zeros(T, torch.int32),
                                 accept_out=zeros(2 + T, torch.int32), workspace=workspace(),
                                 stream=STREAM)
    assert e.value.status == 1
    bad_tree = np.array([-1, 0, 5] + list(range(2, T - 1)), np.int32)
    with pytest.raises(L.TsError) as e:
        L.tree_verify_attn(*_attn_inputs(), N_CTX, bad_tree, out=zeros((T, HQ, D)),
                           workspace=workspace(), stream=STREAM)
    assert e.value.status == 1
