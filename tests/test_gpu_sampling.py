"""GPU parity of the penalty/acceptance options and of the commit of the
accepted path, through the C ABI, against the fp64/binary32 oracle.

* TS_PENALIZE_PATH_TOKENS: each node's draft-path tokens join its penalty
  window (aiboss88, "Contextual penalty strategy");
* TS_ACCEPT_RANDOM_TIE: the kept node is the (r mod c)-th of the c deepest
  valid nodes (aiboss88, tree-based verification: "randomly selected");
* ts_penalize_sample_accept: temperature acceptance, each node's target
  token the Gumbel-max draw from softmax(penalised / temperature) with
  caller-drawn noise (aiboss88, tree-based verification: lossless, with
  diversity);
* ts_kv_commit_path: the accepted path's tree rows move to the context end
  (tencent, parallel-verification figure).

All integer results are compared exactly: argmax, draws, accepted length,
bonus, path, and the committed cache rows bit for bit.
"""
import ctypes
import json
import os

import numpy as np
import pytest
import torch

import lossless_ultra_long_b200 as L
from lossless_ultra_long_b200 import inputs as I
from helpers import dev_bf16, dev_f32, dev_i32, host_bits

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "sampling_cases.json")
PATH, RAND = L.TS_PENALIZE_PATH_TOKENS, L.TS_ACCEPT_RANDOM_TIE


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L.library()


def run_pen(logits, window, penalty, parent, tokens, flags, r=0):
    acc, am = L.penalize_accept(dev_f32(logits), dev_i32(window), penalty, parent,
                                dev_i32(tokens), flags=flags, random=r)
    torch.cuda.synchronize()
    return acc.cpu().numpy(), am.cpu().numpy()


def test_path_window_golden_cases():
    for c in json.load(open(GOLDEN))["path_window"]:
        lg = np.array(c["logits"], np.float32)
        _, am = run_pen(lg, np.array(c["window"], np.int32), c["penalty"], c["parent"],
                        c["tokens"], PATH)
        np.testing.assert_array_equal(am, c["argmax_with_path"], err_msg=c["name"])


@pytest.mark.parametrize("w", [I.TINY, I.LLAMA8B_32K, I.MHA7B_100K], ids=lambda w: w.name)
def test_path_window_workloads(oracle_mod, w):
    """The workloads' logits with the draft tokens drawn among each node's
    top candidates, so that the path tokens change some decisions."""
    parent = w.parent()
    lg = I.gen_logits(w)
    win = I.gen_window(w)
    tokens, lg = I.gen_tree_tokens(w, parent, lg)
    # draft tokens that are strong candidates at their own node: the id of
    # each node's largest logit (so its penalty moves that node's argmax)
    tokens[1:] = np.argmax(lg[1:], axis=1).astype(np.int32)
    acc, am = run_pen(lg, win, w.penalty, parent, tokens, PATH)
    want_am = oracle_mod.penalize_argmax_path(lg, win, parent, tokens, w.penalty)
    np.testing.assert_array_equal(am, want_am)
    assert (want_am != oracle_mod.penalize_argmax(lg, win, w.penalty)).any()
    np.testing.assert_array_equal(acc, oracle_mod.accept_longest(parent, tokens, want_am))


def test_random_tie_golden_case():
    c = json.load(open(GOLDEN))["random_tie"]
    t = len(c["parent"])
    lg = np.full((t, 64), -1.0, np.float32)
    for i, a in enumerate(c["argmax"]):
        lg[i, a] = 1.0
    for r, exp in c["expected"].items():
        acc, _ = run_pen(lg, np.zeros(0, np.int32), 1.2, c["parent"], c["tokens"], RAND, int(r))
        np.testing.assert_array_equal(acc[: len(exp)], exp, err_msg=r)
        assert np.all(acc[len(exp):] == -1)


def test_random_tie_many_equal_paths(oracle_mod):
    """A 40-node 3-ary tree whose siblings all carry the parent's argmax:
    every node is valid and the 27 leaves tie; every r in [0, 60) and a few
    large ones against the oracle, and each leaf is reached."""
    parent = I.bfs_tree(40)
    t, vocab = 40, 1000
    rng = np.random.default_rng(31)
    am = rng.integers(0, vocab, size=t).astype(np.int32)
    lg = rng.normal(0, 2, size=(t, vocab)).astype(np.float32)
    lg[np.arange(t), am] = 50.0
    tokens = np.zeros(t, np.int32)
    tokens[1:] = am[parent[1:]]
    ends = set()
    for r in list(range(60)) + [2 ** 63 + 5, 2 ** 64 - 1, 123456789012345]:
        acc, got_am = run_pen(lg, np.zeros(0, np.int32), 1.2, parent, tokens, RAND | PATH, r)
        want_am = oracle_mod.penalize_argmax_path(lg, np.zeros(0, np.int32), parent, tokens, 1.2)
        np.testing.assert_array_equal(got_am, want_am)
        np.testing.assert_array_equal(acc, oracle_mod.accept_longest_random(parent, tokens,
                                                                          want_am, r))
        ends.add(int(acc[2 + acc[0]]))
    if (want_am[parent[1:]] == tokens[1:]).all():
        assert len(ends) == 27


def test_random_tie_zero_equals_deterministic(oracle_mod):
    w = I.LLAMA8B_32K
    parent = w.parent()
    tokens, lg = I.gen_tree_tokens(w, parent, I.gen_logits(w))
    win = I.gen_window(w)
    a0, _ = run_pen(lg, win, w.penalty, parent, tokens, 0)
    a1, _ = run_pen(lg, win, w.penalty, parent, tokens, RAND, 0)
    np.testing.assert_array_equal(a0, a1)


def test_options_reject_unknown_flags():
    lg = dev_f32(np.zeros((2, 8), np.float32))
    with pytest.raises(L.TsError) as e:
        L.penalize_accept(lg, None, 1.2, [-1, 0], dev_i32([0, 0]), flags=4)
    assert e.value.status == 1


def test_path_window_bad_token_sets_status():
    lg = dev_f32(np.zeros((2, 100), np.float32))
    ws = L.new_workspace(L.penalize_accept_workspace_size(2, 100))
    L.penalize_accept(lg, None, 1.2, [-1, 0], dev_i32([0, 100]), workspace=ws, flags=PATH)
    assert L.workspace_status(ws) == 6
    L.penalize_accept(lg, None, 1.2, [-1, 0], dev_i32([0, 99]), workspace=ws, flags=PATH)
    assert L.workspace_status(ws) == 0


# ------------------------------------------------------- temperature draw
def run_sample(logits, gumbel, temperature, window, penalty, parent, tokens, flags=0, r=0):
    acc, tg = L.penalize_sample_accept(dev_f32(logits), dev_f32(gumbel), temperature,
                                       dev_i32(window), penalty, parent, dev_i32(tokens),
                                       flags=flags, random=r)
    torch.cuda.synchronize()
    return acc.cpu().numpy(), tg.cpu().numpy()


def test_temperature_golden_cases():
    t = json.load(open(GOLDEN))["temperature"]
    none = np.zeros(0, np.int32)
    for c in t["draws"]:
        pen = np.array(c["penalized"], np.float32)
        _, tg = run_sample(pen, np.array(c["gumbel"], np.float32), c["temperature"], none, 1.2,
                           I.chain_tree(len(pen)), np.zeros(len(pen), np.int32))
        np.testing.assert_array_equal(tg, c["expected"], err_msg=c["name"])
    c = t["tree"]
    acc, tg = run_sample(np.array(c["penalized"], np.float32), np.array(c["gumbel"], np.float32),
                         c["temperature"], none, 1.2, c["parent"], c["tokens"])
    np.testing.assert_array_equal(tg, c["expected_draws"])
    np.testing.assert_array_equal(acc[:len(c["expected_accept"])], c["expected_accept"])


@pytest.mark.parametrize("temperature", [0.6, 1.0, 1.7])
@pytest.mark.parametrize("w", [I.TINY, I.LLAMA8B_32K, I.MHA7B_100K], ids=lambda w: w.name)
def test_temperature_workloads(oracle_mod, w, temperature):
    """The workloads' logits (planted maxima), window and seeded noise: the
    draws against the oracle's, then tokens re-planted on the oracle's draws
    so that the accepted path runs deep, with and without the random tie."""
    parent = w.parent()
    tokens, lg = I.gen_tree_tokens(w, parent, I.gen_logits(w))
    win = I.gen_window(w)
    g = I.gen_gumbel(w, draw=int(temperature * 10))
    am, pen = oracle_mod.penalize_argmax(lg, win, w.penalty, return_penalized=True)
    want = oracle_mod.sample_targets(pen, g, temperature)
    assert (want != am).any()   # the draw is not the argmax
    acc, tg = run_sample(lg, g, temperature, win, w.penalty, parent, tokens)
    np.testing.assert_array_equal(tg, want)
    np.testing.assert_array_equal(acc, oracle_mod.accept_longest(parent, tokens, want))
    # every child carries its parent's draw: every node is valid, the leaves tie
    deep = tokens.copy()
    deep[1:] = want[parent[1:]]
    for r in (0, 1, 7, 2 ** 64 - 1):
        acc, tg = run_sample(lg, g, temperature, win, w.penalty, parent, deep, RAND, r)
        np.testing.assert_array_equal(tg, want)
        np.testing.assert_array_equal(acc, oracle_mod.accept_longest_random(parent, deep, want, r))
    depth = np.zeros(len(parent), np.int64)
    for i in range(1, len(parent)):
        depth[i] = depth[parent[i]] + 1
    assert acc[0] == depth.max()


def test_temperature_with_path_window(oracle_mod):
    w = I.LLAMA8B_32K
    parent = w.parent()
    lg = I.gen_logits(w)
    win = I.gen_window(w)
    tokens, lg = I.gen_tree_tokens(w, parent, lg)
    tokens[1:] = np.argmax(lg[1:], axis=1).astype(np.int32)
    g = I.gen_gumbel(w, draw=3)
    _, pen = oracle_mod.penalize_argmax_path(lg, win, parent, tokens, w.penalty,
                                             return_penalized=True)
    want = oracle_mod.sample_targets(pen, g, 0.8)
    acc, tg = run_sample(lg, g, 0.8, win, w.penalty, parent, tokens, PATH)
    np.testing.assert_array_equal(tg, want)
    np.testing.assert_array_equal(acc, oracle_mod.accept_longest(parent, tokens, want))


def test_temperature_one_without_noise_is_the_argmax_call(oracle_mod):
    w = I.LLAMA8B_32K
    parent = w.parent()
    tokens, lg = I.gen_tree_tokens(w, parent, I.gen_logits(w))
    win = I.gen_window(w)
    acc, tg = run_sample(lg, np.zeros_like(lg), 1.0, win, w.penalty, parent, tokens)
    acc0, am0 = run_pen(lg, win, w.penalty, parent, tokens, 0)
    np.testing.assert_array_equal(tg, am0)
    np.testing.assert_array_equal(acc, acc0)
    np.testing.assert_array_equal(tg, oracle_mod.penalize_argmax(lg, win, w.penalty))


def test_temperature_ragged_vocab_and_nan(oracle_mod):
    """A vocabulary that is not a multiple of 4 (the scalar route), NaN
    logits and NaN noise, against the oracle."""
    rng = np.random.default_rng(51)
    t, vocab = 13, 1001
    parent = I.bfs_tree(t)
    lg = rng.normal(0, 2, size=(t, vocab)).astype(np.float32)
    g = rng.gumbel(size=(t, vocab)).astype(np.float32)
    lg[2, ::7] = np.nan
    g[5, ::3] = np.nan
    win = rng.integers(0, vocab, size=64).astype(np.int32)
    tokens = rng.integers(0, vocab, size=t).astype(np.int32)
    _, pen = oracle_mod.penalize_argmax(lg, win, 1.3, return_penalized=True)
    want = oracle_mod.sample_targets(pen, g, 1.4)
    tokens[1:] = want[parent[1:]]
    acc, tg = run_sample(lg, g, 1.4, win, 1.3, parent, tokens)
    np.testing.assert_array_equal(tg, want)
    np.testing.assert_array_equal(acc, oracle_mod.accept_longest(parent, tokens, want))


def test_temperature_rejects_bad_arguments():
    lib = L.library()
    lg = dev_f32(np.zeros((2, 8), np.float32))
    g = dev_f32(np.zeros((2, 12), np.float32))
    tok = dev_i32([0, 0])
    acc = torch.empty(4, dtype=torch.int32, device="cuda")
    ws = L.new_workspace(L.penalize_accept_workspace_size(2, 8))
    par = np.array([-1, 0], np.int32)
    P = ctypes.c_void_p

    def call(gptr, temp):
        return lib.ts_penalize_sample_accept(
            P(lg.data_ptr()), gptr, temp, 2, 8, None, 0, 1.2, par.ctypes.data_as(P),
            P(tok.data_ptr()), 0, 0, None, P(acc.data_ptr()), P(ws.data_ptr()), ws.numel(), None)

    assert call(P(g.data_ptr()), 1.0) == 0
    torch.cuda.synchronize()
    assert call(None, 1.0) == 1
    assert call(P(g.data_ptr() + 4), 1.0) == 1     # not 16-byte aligned
    for bad in (0.0, -0.5, float("inf"), float("nan")):
        assert call(P(g.data_ptr()), bad) == 1


# ------------------------------------------------------------------ commit
def test_commit_golden_case():
    c = json.load(open(GOLDEN))["commit"]
    rows = np.array(c["rows"], np.uint16)
    # D must be 64 or 128: the fixture's two columns, repeated
    k = np.tile(rows, (1, 64))[None]
    v = (np.tile(rows, (1, 64)) + 1)[None].astype(np.uint16)
    dk, dv = dev_bf16(k), dev_bf16(v)
    L.kv_commit_path(dk, dv, c["n_ctx"], c["n_tree"], dev_i32(c["accept"]))
    torch.cuda.synchronize()
    want = np.tile(np.array(c["expected_rows"], np.uint16), (1, 64))
    np.testing.assert_array_equal(host_bits(dk)[0], want)
    np.testing.assert_array_equal(host_bits(dv)[0], want + 1)


@pytest.mark.parametrize("hkv,d,n_ctx,t", [(8, 128, 32768, 40), (2, 64, 2048, 13),
                                           (32, 128, 1000, 64), (8, 128, 0, 4)])
def test_commit_matches_oracle(oracle_mod, hkv, d, n_ctx, t):
    rng = np.random.default_rng(n_ctx + t)
    cap = n_ctx + t + 7
    k = rng.integers(0, 65535, size=(hkv, cap, d)).astype(np.uint16)
    v = rng.integers(0, 65535, size=(hkv, cap, d)).astype(np.uint16)
    parent = I.bfs_tree(t) if t > 4 else I.chain_tree(t)
    for end in sorted({0, t - 1, int(rng.integers(0, t))}):
        path, a = [], end
        while a >= 0:
            path.append(a)
            a = int(parent[a])
        path.reverse()
        acc = np.full(2 + t, -1, np.int32)
        acc[0], acc[1] = len(path) - 1, 5
        acc[2:2 + len(path)] = path
        dk, dv = dev_bf16(k), dev_bf16(v)
        L.kv_commit_path(dk, dv, n_ctx, t, dev_i32(acc))
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host_bits(dk), oracle_mod.kv_commit_path(k, n_ctx, t, acc))
        np.testing.assert_array_equal(host_bits(dv), oracle_mod.kv_commit_path(v, n_ctx, t, acc))


def test_accept_then_commit_on_the_device(oracle_mod):
    """penalize_accept and the commit on one stream, no host round trip: the
    cache afterwards is the oracle's commit of the oracle's acceptance."""
    w = I.LLAMA8B_32K.with_(n_ctx=4096)
    parent = w.parent()
    tokens, lg = I.gen_tree_tokens(w, parent, I.gen_logits(w))
    win = I.gen_window(w)
    k, v = I.gen_kv(w)
    dk, dv = dev_bf16(k), dev_bf16(v)
    acc, _ = L.penalize_accept(dev_f32(lg), dev_i32(win), w.penalty, parent, dev_i32(tokens))
    L.kv_commit_path(dk, dv, w.n_ctx, w.n_tree, acc)
    torch.cuda.synchronize()
    want_acc = oracle_mod.accept_longest(parent, tokens,
                                         oracle_mod.penalize_argmax(lg, win, w.penalty))
    np.testing.assert_array_equal(acc.cpu().numpy(), want_acc)
    assert want_acc[0] > 0
    np.testing.assert_array_equal(host_bits(dk), oracle_mod.kv_commit_path(k, w.n_ctx, w.n_tree,
                                                                           want_acc))
    np.testing.assert_array_equal(host_bits(dv), oracle_mod.kv_commit_path(v, w.n_ctx, w.n_tree,
                                                                           want_acc))


def test_commit_rejects_a_result_that_is_not_a_path():
    k = torch.zeros((2, 50, 64), dtype=torch.bfloat16, device="cuda")
    v = torch.ones((2, 50, 64), dtype=torch.bfloat16, device="cuda")
    ws = L.new_workspace(256)
    for bad in ([3, 0, 0, 1, 2, 9, -1], [1, 0, 1, 1, -1, -1, -1], [2, 0, 0, 3, 2, -1, -1],
                [9, 0, 0, 1, 2, 3, 4]):
        L.kv_commit_path(k, v, 40, 5, dev_i32(bad), workspace=ws)
        assert L.workspace_status(ws) == 6, bad
    assert (k == 0).all() and (v == 1).all()
    with pytest.raises(L.TsError) as e:
        L.kv_commit_path(k, v, 46, 5, dev_i32([0, 0, 0, -1, -1, -1, -1]))
    assert e.value.status == 1
