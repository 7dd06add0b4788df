"""The benchmarked verification step, call for call, against the fp64 oracle.

``bench.py`` times one step of the path on the LLaMA3.1-8B 100K-context
workload (spiked keys): the verify attention that also leaves the root
node's scores, the sink + top-budget select on those scores with the gather
into the partial cache, the draft pass over that gathered cache, the
penalty/argmax/acceptance call on a second stream, and the commit of the
accepted path's K/V rows.  This test builds the
very same ``Step`` object, runs one step exactly as the benchmark does
(both streams), and checks every stage:

* verify attention: all 32 rows of the root node and 96 sampled rows,
  max |err| <= 2e-3 against the oracle;
* root scores (base 2) at every context position against fp64 products;
* importance scores at every position, relative error <= 1e-3;
* kept indices: exactly the oracle's sink + top-budget of the GPU's scores;
* gathered K/V rows: bit-identical to the source rows;
* draft pass: the oracle's attention over the gathered cache (all rows);
* penalised argmax and the accepted path: exact;
* the commit of the accepted path: the tree-tail rows, bit for bit.
"""
import os
import sys

import numpy as np
import pytest
import torch

import lossless_ultra_long_b200 as L
from lossless_ultra_long_b200 import inputs as I
from helpers import host_bits, sample_rows

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ATTN_TOL = 2e-3
SCORE_RTOL = 1e-3


@pytest.fixture(scope="module")
def step_result():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sys.path.insert(0, ROOT)
    import bench
    L.library()
    w = bench.workload()
    assert w is I.LLAMA8B_100K
    st = bench.Step(torch, L, I, w, torch.device("cuda", 0), fused=True, want_scores=True)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        st.step()
    stream.synchronize()
    torch.cuda.synchronize()
    return st


@pytest.fixture(scope="module")
def host_inputs(step_result):
    """The step's seeded inputs as the oracle reads them (bf16 bit patterns)."""
    w = step_result.w
    k, v = I.gen_kv(w)
    return I.gen_q(w), k, v


def test_step_verify_attention(oracle_mod, step_result, host_inputs):
    st, w = step_result, step_result.w
    q, k, v = host_inputs
    nodes, heads = sample_rows(w.n_tree, w.n_heads_q, 92, 2024)
    nodes = np.concatenate([np.zeros(w.n_heads_q, np.int32), nodes])
    heads = np.concatenate([np.arange(w.n_heads_q, dtype=np.int32), heads])
    want = oracle_mod.tree_verify_attn_rows(q, k, v, w.n_ctx, w.parent(), nodes, heads)
    got = st.out.cpu().numpy().astype(np.float64)
    err = np.abs(got[nodes, heads] - want).max()
    assert err <= ATTN_TOL, f"verify attention max abs err {err}"
    assert np.isfinite(got).all()


def test_step_root_scores(step_result, host_inputs):
    st, w = step_result, step_result.w
    q, k, _ = host_inputs
    qf = I.bf16_bits_to_f32(q[0]).astype(np.float64)
    kf = I.bf16_bits_to_f32(k[:, : w.n_ctx]).astype(np.float64)
    g = np.arange(w.n_heads_q) // w.group
    want = np.einsum("hd,hpd->hp", qf, kf[g]) / np.sqrt(w.head_dim) * np.log2(np.e)
    got = st.rs.cpu().numpy().astype(np.float64)
    assert np.abs(got - want).max() <= 1e-3 * (1.0 + np.abs(want).max())


def test_step_select_and_gather(oracle_mod, step_result, host_inputs):
    st, w = step_result, step_result.w
    q, k, v = host_inputs
    sc = st.scores.cpu().numpy()
    want_sc = oracle_mod.importance_scores(q[0], k, w.n_ctx, w.n_heads_q)
    rel = np.abs(sc - want_sc) / np.maximum(want_sc, 1e-30)
    assert rel.max() <= SCORE_RTOL, f"importance rel err {rel.max()}"
    idx = st.idx.cpu().numpy()
    np.testing.assert_array_equal(idx, oracle_mod.select_topk(sc.astype(np.float64), w.n_sink,
                                                              w.budget))
    kp = host_bits(st.kp)[:, : st.n_keep]
    vp = host_bits(st.vp)[:, : st.n_keep]
    np.testing.assert_array_equal(kp, oracle_mod.gather_rows(k, idx))
    np.testing.assert_array_equal(vp, oracle_mod.gather_rows(v, idx))
    n_keep = w.n_sink + w.budget
    assert idx.shape == (w.n_heads_kv, n_keep)
    for g in range(w.n_heads_kv):
        assert np.all(np.diff(idx[g]) > 0)
        assert set(range(w.n_sink)) <= set(idx[g].tolist())


def test_step_draft_pass_over_gathered_cache(oracle_mod, step_result):
    st, w = step_result, step_result.w
    kp, vp = host_bits(st.kp), host_bits(st.vp)   # gathered rows + the chain's own rows
    want = oracle_mod.tree_verify_attn(I.gen_draft_q(w), kp, vp, st.n_keep,
                                       I.chain_tree(w.draft_tree))
    err = np.abs(st.dout.cpu().numpy().astype(np.float64) - want).max()
    assert err <= ATTN_TOL, f"draft attention max abs err {err}"


def test_step_penalty_and_accept(oracle_mod, step_result):
    st, w = step_result, step_result.w
    parent = w.parent()
    tokens, lg = I.gen_tree_tokens(w, parent, I.gen_logits(w))
    want_am = oracle_mod.penalize_argmax(lg, I.gen_window(w), w.penalty)
    np.testing.assert_array_equal(st.argmax.cpu().numpy(), want_am)
    np.testing.assert_array_equal(st.accept.cpu().numpy(),
                                  oracle_mod.accept_longest(parent, tokens, want_am))


def test_step_commit_of_the_accepted_path(oracle_mod, step_result, host_inputs):
    """After the step the tree-tail rows hold the accepted path in order
    (the rows the verify call read are the seeded ones)."""
    st, w = step_result, step_result.w
    _, k, v = host_inputs
    acc = st.accept.cpu().numpy()
    assert acc[0] >= 1   # the planted tokens make some path valid
    lo, hi = w.n_ctx, w.n_ctx + w.n_tree
    for dev_cache, host in ((st.k, k), (st.v, v)):
        tail = np.ascontiguousarray(host[:, lo:hi])
        want = oracle_mod.kv_commit_path(tail, 0, w.n_tree, acc)
        np.testing.assert_array_equal(host_bits(dev_cache[:, lo:hi].contiguous()), want)
