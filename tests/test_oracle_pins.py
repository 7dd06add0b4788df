"""Pins of the fp64 CPU oracle against what the TokenSwift pages and plain
mathematics fix, independently of the oracle's own code.

Each test ties one oracle function to something other than itself: a
library routine (torch's scaled-dot-product attention, torch.softmax), a
brute-force restatement on tiny inputs, a closed form, an invariant, or a
hand-worked fixture under tests/golden/ citing the passage it follows.
"""
import json
import os

import numpy as np
import pytest
import torch

from lossless_ultra_long_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f64(bits):
    return I.bf16_bits_to_f32(bits).astype(np.float64)


def _small(seed, hq=4, hkv=2, d=16, n_ctx=37, t=13, tree="ternary"):
    w = I.Workload("pin", hq, hkv, d, n_ctx, t, tree=tree, seed=seed)
    q = I.gen_q(w)
    k, v = I.gen_kv(w)
    return w, q, k, v


# ------------------------------------------------------------------ attention
def test_single_node_tree_equals_library_decode(oracle_mod):
    """T = 1 is ordinary decode: torch SDPA (fp64, no mask, GQA by repeat)."""
    w, q, k, v = _small(10, hq=8, hkv=2, d=64, n_ctx=300, t=1)
    out = oracle_mod.tree_verify_attn(q, k, v, w.n_ctx, w.parent())
    Q = torch.from_numpy(_f64(q))                       # [1, Hq, D]
    K = torch.from_numpy(_f64(k[:, : w.n_ctx + 1]))      # [Hkv, N+1, D]
    V = torch.from_numpy(_f64(v[:, : w.n_ctx + 1]))
    K = K.repeat_interleave(w.group, dim=0)              # head h -> kv head h // G
    V = V.repeat_interleave(w.group, dim=0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.permute(1, 0, 2), K, V, scale=1.0 / np.sqrt(w.head_dim))
    np.testing.assert_allclose(out, ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


def _bruteforce_path_attention(q, k, v, n_ctx, parent, scale):
    """Dense attention of each node over its explicit token sequence."""
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    t, hq, d = qf.shape
    hkv = kf.shape[0]
    out = np.zeros((t, hq, d))
    for i in range(t):
        path = []
        a = i
        while a >= 0:
            path.append(a)
            a = int(parent[a])
        seq = list(range(n_ctx)) + [n_ctx + a for a in reversed(path)]
        for h in range(hq):
            g = h // (hq // hkv)
            logits = torch.from_numpy(kf[g, seq] @ qf[i, h] * scale)
            p = torch.softmax(logits, dim=0).numpy()
            out[i, h] = p @ vf[g, seq]
    return out


@pytest.mark.parametrize("tree", ["ternary", "chain"])
@pytest.mark.parametrize("t", [1, 4, 13, 40])
def test_tree_mask_equals_bruteforce_paths(oracle_mod, tree, t):
    w, q, k, v = _small(11 + t, hq=6, hkv=3, d=8, n_ctx=29, t=t, tree=tree)
    p = w.parent()
    out = oracle_mod.tree_verify_attn(q, k, v, w.n_ctx, p)
    ref = _bruteforce_path_attention(q, k, v, w.n_ctx, p, 1 / np.sqrt(8))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)


def test_irregular_tree_equals_bruteforce(oracle_mod):
    """A non-complete tree (mixed fan-out) in topological order."""
    parent = np.array([-1, 0, 0, 1, 1, 1, 2, 4, 4, 7, 3, 10], dtype=np.int32)
    w, q, k, v = _small(21, hq=4, hkv=1, d=16, n_ctx=17, t=len(parent))
    out = oracle_mod.tree_verify_attn(q, k, v, w.n_ctx, parent)
    ref = _bruteforce_path_attention(q, k, v, w.n_ctx, parent, 0.25)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)


def test_chain_tree_equals_sequential_decode(oracle_mod):
    """A chain verified in one pass equals T causal decode steps with a growing cache."""
    w, q, k, v = _small(30, hq=8, hkv=2, d=32, n_ctx=50, t=7, tree="chain")
    out = oracle_mod.tree_verify_attn(q, k, v, w.n_ctx, w.parent())
    for i in range(w.n_tree):
        # step i: context = everything before position n_ctx + i, query = node i
        step = oracle_mod.tree_verify_attn(q[i : i + 1], k, v, w.n_ctx + i,
                                           np.array([-1], dtype=np.int32))
        np.testing.assert_allclose(out[i], step[0], rtol=0, atol=1e-13)


def test_uniform_keys_average_exactly_the_visible_values(oracle_mod):
    """Equal keys give equal weights: out = mean of V over the visible set.
    The tail V rows are one-hot markers, so the visible tail set is read off."""
    parent = I.bfs_tree(13)
    hq, hkv, d, n_ctx = 2, 1, 16, 5
    t = len(parent)
    k = np.full((hkv, n_ctx + t, d), I.f32_to_bf16_bits(np.array([0.5], np.float32))[0],
                dtype=np.uint16)
    vf = np.zeros((hkv, n_ctx + t, d), dtype=np.float32)
    vf[0, n_ctx:, :t] = np.eye(t, dtype=np.float32)      # tail row a marks column a
    v = I.f32_to_bf16_bits(vf)
    q = I.gen_q(I.Workload("u", hq, hkv, d, n_ctx, t, seed=3))
    out = oracle_mod.tree_verify_attn(q, k, v, n_ctx, parent)
    for i in range(t):
        path = set()
        a = i
        while a >= 0:
            path.add(a)
            a = int(parent[a])
        n_vis = n_ctx + len(path)
        want = np.array([1.0 / n_vis if c in path else 0.0 for c in range(d)])
        for h in range(hq):
            np.testing.assert_allclose(out[i, h], want, rtol=0, atol=1e-15)


def test_gqa_head_mapping(oracle_mod):
    """Query head h reads KV head h // (Hq/Hkv): KV head g has V constant g+1."""
    hq, hkv, d, n_ctx, t = 12, 3, 8, 9, 4
    parent = I.bfs_tree(t)
    w = I.Workload("g", hq, hkv, d, n_ctx, t, seed=4)
    q = I.gen_q(w)
    k, _ = I.gen_kv(w)
    vf = np.zeros((hkv, n_ctx + t, d), dtype=np.float32)
    for g in range(hkv):
        vf[g] = g + 1
    out = oracle_mod.tree_verify_attn(q, k, I.f32_to_bf16_bits(vf), n_ctx, parent)
    for h in range(hq):
        np.testing.assert_allclose(out[:, h], h // (hq // hkv) + 1, rtol=0, atol=1e-14)


def test_one_visible_position(oracle_mod):
    """Empty context, single node: the output is the root's own V row."""
    w, q, k, v = _small(5, hq=4, hkv=2, d=16, n_ctx=0, t=1)
    out = oracle_mod.tree_verify_attn(q, k, v, 0, w.parent())
    for h in range(4):
        np.testing.assert_array_equal(out[0, h], _f64(v[h // 2, 0]))


def test_rows_entry_matches_full(oracle_mod):
    w, q, k, v = _small(6, hq=8, hkv=4, d=16, n_ctx=20, t=13)
    full = oracle_mod.tree_verify_attn(q, k, v, w.n_ctx, w.parent())
    nodes = np.array([0, 12, 5, 7], dtype=np.int32)
    heads = np.array([7, 0, 3, 4], dtype=np.int32)
    rows = oracle_mod.tree_verify_attn_rows(q, k, v, w.n_ctx, w.parent(), nodes, heads)
    np.testing.assert_array_equal(rows, full[nodes, heads])


def test_attention_rejects_bad_tree(oracle_mod):
    w, q, k, v = _small(7, t=4)
    with pytest.raises(ValueError):
        oracle_mod.tree_verify_attn(q, k, v, w.n_ctx, np.array([-1, 0, 3, 1], np.int32))
    with pytest.raises(ValueError):
        oracle_mod.tree_verify_attn(q, k, v, w.n_ctx, np.array([0, 0, 1, 1], np.int32))


# ----------------------------------------------------------------- importance
def test_importance_single_head_group_is_library_softmax(oracle_mod):
    w, q, k, v = _small(40, hq=3, hkv=3, d=32, n_ctx=100, t=1)
    s = oracle_mod.importance_scores(q[0], k, w.n_ctx, 3)
    for g in range(3):
        logits = torch.from_numpy(_f64(k[g, : w.n_ctx]) @ _f64(q[0, g]) / np.sqrt(32))
        np.testing.assert_allclose(s[g], torch.softmax(logits, 0).numpy(), rtol=1e-13, atol=0)


def test_importance_is_group_mean_of_softmaxes(oracle_mod):
    """G = 4: scores are the mean of four per-head softmaxes; each sums to 1."""
    w, q, k, v = _small(41, hq=8, hkv=2, d=16, n_ctx=64, t=1)
    s = oracle_mod.importance_scores(q[0], k, w.n_ctx, 8)
    np.testing.assert_allclose(s.sum(1), 1.0, rtol=0, atol=1e-13)
    for g in range(2):
        probs = []
        for h in range(4 * g, 4 * g + 4):
            logits = torch.from_numpy(_f64(k[g, : w.n_ctx]) @ _f64(q[0, h]) / 4.0)
            probs.append(torch.softmax(logits, 0).numpy())
        np.testing.assert_allclose(s[g], np.mean(probs, 0), rtol=1e-13, atol=0)


def test_importance_excludes_tree_tail(oracle_mod):
    """Rows past n_ctx do not enter the softmax."""
    w, q, k, v = _small(42, hq=2, hkv=1, d=16, n_ctx=30, t=5)
    s1 = oracle_mod.importance_scores(q[0], k, 30, 2)
    k2 = k.copy()
    k2[:, 30:] = 0x4500  # large keys in the tail
    s2 = oracle_mod.importance_scores(q[0], k2, 30, 2)
    np.testing.assert_array_equal(s1, s2)


# ------------------------------------------------------------------- top-k
def _brute_select(scores, n_sink, budget):
    hkv, n = scores.shape
    out = []
    for g in range(hkv):
        if n <= n_sink + budget:
            out.append(list(range(n)))
            continue
        cand = sorted(range(n_sink, n), key=lambda j: (-scores[g, j], j))[:budget]
        out.append(sorted(list(range(n_sink)) + cand))
    return np.array(out, dtype=np.int32)


@pytest.mark.parametrize("n_sink,budget", [(4, 10), (0, 7), (16, 0), (3, 100), (50, 50)])
def test_select_matches_bruteforce_with_ties(oracle_mod, n_sink, budget):
    rng = np.random.default_rng(7)
    scores = rng.integers(0, 6, size=(3, 97)).astype(np.float64) / 8.0  # many exact ties
    idx = oracle_mod.select_topk(scores, n_sink, budget)
    np.testing.assert_array_equal(idx, _brute_select(scores, n_sink, budget))


def test_select_invariants(oracle_mod):
    rng = np.random.default_rng(8)
    scores = rng.random((4, 500))
    idx = oracle_mod.select_topk(scores, 16, 240)
    assert idx.shape == (4, 256)
    for g in range(4):
        assert np.all(np.diff(idx[g]) > 0)
        assert set(range(16)) <= set(idx[g].tolist())
        kept = idx[g][16:]
        thresh = scores[g, kept].min()
        others = np.setdiff1d(np.arange(16, 500), kept)
        assert np.all(scores[g, others] <= thresh)


def test_select_uniform_scores_take_lowest_positions(oracle_mod):
    idx = oracle_mod.select_topk(np.full((2, 50), 0.02), 5, 10)
    np.testing.assert_array_equal(idx, np.tile(np.arange(15, dtype=np.int32), (2, 1)))


def test_select_spikes_are_found(oracle_mod):
    """Keys with a large planted score are exactly the selected set."""
    scores = np.full((1, 200), 1e-3)
    planted = [17, 44, 45, 150, 199]
    scores[0, planted] = 0.5
    scores[0, 2] = 0.9   # a sink: kept anyway, not counted against the budget
    idx = oracle_mod.select_topk(scores, 4, 5)
    np.testing.assert_array_equal(idx[0], [0, 1, 2, 3] + planted)


def test_gather_copies_rows_bit_exactly(oracle_mod):
    w, q, k, v = _small(9, hq=2, hkv=2, d=16, n_ctx=40, t=1)
    idx = np.array([[0, 3, 9, 39], [1, 2, 20, 30]], dtype=np.int32)
    kp = oracle_mod.gather_rows(k, idx, partial_cap=6)
    for g in range(2):
        np.testing.assert_array_equal(kp[g, :4], k[g, idx[g]])
        assert not kp[g, 4:].any()


# ---------------------------------------------------------- penalty + argmax
def test_penalty_golden_cases(oracle_mod):
    cases = json.load(open(os.path.join(GOLDEN, "penalty_cases.json")))["cases"]
    for c in cases:
        lg = np.array(c["logits"], dtype=np.float32)
        am, pen = oracle_mod.penalize_argmax(lg, np.array(c["window"], np.int32), c["penalty"],
                                             return_penalized=True)
        np.testing.assert_array_equal(pen.view(np.uint32),
                                      np.array(c["penalized"], np.float32).view(np.uint32),
                                      err_msg=c["name"])
        np.testing.assert_array_equal(am, c["argmax"], err_msg=c["name"])


def test_penalty_nan_is_never_the_argmax(oracle_mod):
    lg = np.array([[np.nan, 1.0, -3.0], [np.nan, np.nan, np.nan], [-np.inf, -np.inf, 2.0]],
                  np.float32)
    am = oracle_mod.penalize_argmax(lg, np.array([], np.int32), 1.2)
    np.testing.assert_array_equal(am, [1, 0, 2])


def test_penalty_rejects_out_of_vocab_window(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.penalize_argmax(np.zeros((1, 8), np.float32), np.array([8], np.int32), 1.2)


def test_penalty_12_matches_ieee_binary32():
    """Penalty 1.2f: the oracle's result equals numpy's binary32 division and product."""
    import oracle
    rng = np.random.default_rng(3)
    lg = rng.normal(0, 2, size=(3, 1000)).astype(np.float32)
    win = np.arange(0, 1000, 3, dtype=np.int32)
    _, pen = oracle.penalize_argmax(lg, win, 1.2, return_penalized=True)
    p = np.float32(1.2)
    for i in range(3):
        for j in (0, 3, 6, 999):
            x = lg[i, j]
            want = np.float32(x / p) if x > 0 else np.float32(x * p)
            assert pen[i, j].view(np.uint32) == want.view(np.uint32)
        assert pen[i, 1] == lg[i, 1]


# --------------------------------------------------------------- acceptance
def test_accept_golden_cases(oracle_mod):
    cases = json.load(open(os.path.join(GOLDEN, "accept_cases.json")))["cases"]
    for c in cases:
        out = oracle_mod.accept_longest(c["parent"], c["tokens"], c["argmax"])
        exp = c["expected"]
        np.testing.assert_array_equal(out[: len(exp)], exp, err_msg=c["name"])
        assert np.all(out[len(exp):] == -1), c["name"]


def test_accept_figure_example(oracle_mod):
    """'is the father of' from the tencent figure text, end to end through the
    penalty + argmax + acceptance oracles."""
    f = json.load(open(os.path.join(GOLDEN, "accept_figure.json")))
    t = len(f["parent"])
    lg = np.full((t, f["vocab"]), -1.0, dtype=np.float32)
    for node, tok in f["target_argmax_at_node"].items():
        lg[int(node), tok] = 5.0
    am = oracle_mod.penalize_argmax(lg, np.array(f["window"], np.int32), f["penalty"])
    out = oracle_mod.accept_longest(f["parent"], f["tokens"], am)
    exp = f["expected_accept"]
    np.testing.assert_array_equal(out[: len(exp)], exp)
    words = [f["vocab_names"][f["tokens"][n]] for n in out[3 : 2 + exp[0] + 1]]
    assert " ".join(words) == "is the father of"


def test_accept_matches_exhaustive_path_search(oracle_mod):
    """Random trees: the result equals the longest root path, over all paths, whose
    every step matches the parent's argmax (lowest end node on equal length)."""
    rng = np.random.default_rng(12)
    for trial in range(200):
        t = int(rng.integers(1, 30))
        parent = np.array([-1] + [int(rng.integers(0, i)) for i in range(1, t)], np.int32)
        tokens = rng.integers(0, 3, size=t).astype(np.int32)
        argmax = rng.integers(0, 3, size=t).astype(np.int32)
        best_len, best_end = 0, 0
        for end in range(t):
            path = []
            a = end
            while a >= 0:
                path.append(a)
                a = int(parent[a])
            path.reverse()
            ok = all(tokens[path[s + 1]] == argmax[path[s]] for s in range(len(path) - 1))
            if ok and len(path) - 1 > best_len:
                best_len, best_end = len(path) - 1, end
        out = oracle_mod.accept_longest(parent, tokens, argmax)
        assert out[0] == best_len and out[1] == argmax[best_end], trial
        assert out[2 + best_len] == best_end


# ------------------------------------------------- sampling variants, commit
SAMPLING = os.path.join(GOLDEN, "sampling_cases.json")


def test_path_window_golden_cases(oracle_mod):
    for c in json.load(open(SAMPLING))["path_window"]:
        lg = np.array(c["logits"], np.float32)
        win = np.array(c["window"], np.int32)
        am = oracle_mod.penalize_argmax_path(lg, win, c["parent"], c["tokens"], c["penalty"])
        np.testing.assert_array_equal(am, c["argmax_with_path"], err_msg=c["name"])
        np.testing.assert_array_equal(oracle_mod.penalize_argmax(lg, win, c["penalty"]),
                                      c["argmax_window_only"], err_msg=c["name"])


def test_path_window_is_the_window_with_each_path_added(oracle_mod):
    """Per node, the result equals the plain penalty run with that node's
    window widened by its draft-path tokens (collected here by walking the
    parents), on random trees with small vocabularies (many collisions)."""
    rng = np.random.default_rng(21)
    for trial in range(40):
        t = int(rng.integers(1, 20))
        vocab = int(rng.integers(2, 40))
        parent = np.array([-1] + [int(rng.integers(0, i)) for i in range(1, t)], np.int32)
        tokens = rng.integers(0, vocab, size=t).astype(np.int32)
        win = rng.integers(0, vocab, size=int(rng.integers(0, 8))).astype(np.int32)
        lg = rng.normal(0, 2, size=(t, vocab)).astype(np.float32)
        am = oracle_mod.penalize_argmax_path(lg, win, parent, tokens, 1.2)
        for i in range(t):
            path, a = [], i
            while a != 0:
                path.append(int(tokens[a]))
                a = int(parent[a])
            wi = np.concatenate([win, np.array(path, np.int32)])
            assert am[i] == oracle_mod.penalize_argmax(lg[i:i + 1], wi, 1.2)[0], (trial, i)


def test_path_window_single_node_equals_plain_penalty(oracle_mod):
    rng = np.random.default_rng(22)
    lg = rng.normal(0, 2, size=(1, 500)).astype(np.float32)
    win = rng.integers(0, 500, size=50).astype(np.int32)
    np.testing.assert_array_equal(
        oracle_mod.penalize_argmax_path(lg, win, [-1], [7], 1.2),
        oracle_mod.penalize_argmax(lg, win, 1.2))


def test_path_window_rejects_out_of_vocab_tokens(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.penalize_argmax_path(np.zeros((2, 8), np.float32), np.zeros(0, np.int32),
                                        [-1, 0], [0, 8], 1.2)


def test_random_tie_golden_case(oracle_mod):
    c = json.load(open(SAMPLING))["random_tie"]
    for r, exp in c["expected"].items():
        out = oracle_mod.accept_longest_random(c["parent"], c["tokens"], c["argmax"], int(r))
        np.testing.assert_array_equal(out[: len(exp)], exp, err_msg=r)
        assert np.all(out[len(exp):] == -1)


def test_random_tie_matches_exhaustive_path_search(oracle_mod):
    """Random trees with few token values (many equally long valid paths):
    for every r the kept path is the (r mod c)-th, in end-node order, of the
    c longest root paths whose every step matches the parent's argmax, and
    r = 0 is the deterministic lowest-index rule."""
    rng = np.random.default_rng(23)
    for trial in range(150):
        t = int(rng.integers(1, 25))
        parent = np.array([-1] + [int(rng.integers(0, i)) for i in range(1, t)], np.int32)
        tokens = rng.integers(0, 2, size=t).astype(np.int32)
        argmax = rng.integers(0, 2, size=t).astype(np.int32)
        ends = {}
        for end in range(t):
            path, a = [], end
            while a >= 0:
                path.append(a)
                a = int(parent[a])
            path.reverse()
            if all(tokens[path[s + 1]] == argmax[path[s]] for s in range(len(path) - 1)):
                ends.setdefault(len(path) - 1, []).append(end)
        best_len = max(ends)
        best = sorted(ends[best_len])
        for r in range(2 * len(best) + 1):
            out = oracle_mod.accept_longest_random(parent, tokens, argmax, r)
            end = best[r % len(best)]
            assert out[0] == best_len and out[1] == argmax[end] and out[2 + best_len] == end
        np.testing.assert_array_equal(oracle_mod.accept_longest_random(parent, tokens, argmax, 0),
                                      oracle_mod.accept_longest(parent, tokens, argmax))


def test_temperature_golden_cases(oracle_mod):
    t = json.load(open(SAMPLING))["temperature"]
    for c in t["draws"]:
        got = oracle_mod.sample_targets(np.array(c["penalized"], np.float32),
                                        np.array(c["gumbel"], np.float32), c["temperature"])
        np.testing.assert_array_equal(got, c["expected"], err_msg=c["name"])
    c = t["tree"]
    pen = np.array(c["penalized"], np.float32)
    draws = oracle_mod.sample_targets(pen, np.array(c["gumbel"], np.float32), c["temperature"])
    np.testing.assert_array_equal(draws, c["expected_draws"])
    out = oracle_mod.accept_longest(c["parent"], c["tokens"], draws)
    np.testing.assert_array_equal(out[:len(c["expected_accept"])], c["expected_accept"])
    greedy = oracle_mod.accept_longest(c["parent"], c["tokens"], np.argmax(pen, axis=1))
    np.testing.assert_array_equal(greedy[:len(c["greedy_accept"])], c["greedy_accept"])


@pytest.mark.parametrize("temperature", [0.5, 2.0])
def test_temperature_draws_follow_the_tempered_softmax(oracle_mod, temperature):
    """Gumbel-max: with independent standard Gumbel noise, the draw of each
    row is distributed as softmax(logits / temperature).  200,000 rows of the
    same five logits; every id's frequency within five standard errors of
    the closed-form probability (numpy's own Gumbel generator, fp64
    softmax)."""
    n = 200_000
    logits = np.array([1.0, 0.5, -0.3, 2.0, 1.2], np.float32)
    g = np.random.default_rng(41).gumbel(size=(n, 5)).astype(np.float32)
    draws = oracle_mod.sample_targets(np.tile(logits, (n, 1)), g, temperature)
    z = logits.astype(np.float64) / temperature
    p = np.exp(z - z.max())
    p /= p.sum()
    freq = np.bincount(draws, minlength=5) / n
    se = np.sqrt(p * (1 - p) / n)
    assert np.all(np.abs(freq - p) <= 5 * se + 1e-12), (freq, p)


def test_temperature_one_without_noise_is_the_argmax(oracle_mod):
    """temperature 1 divides exactly and zero noise adds nothing: the draw
    is the penalised argmax (ties to the lowest id), on a workload's logits."""
    w = I.TINY
    lg = I.gen_logits(w)
    lg[3, 17] = lg[3, 5] = 40.0   # a tie
    am, pen = oracle_mod.penalize_argmax(lg, I.gen_window(w), w.penalty, return_penalized=True)
    np.testing.assert_array_equal(oracle_mod.sample_targets(pen, np.zeros_like(pen), 1.0), am)
    assert am[3] == 5


def test_temperature_nan_is_never_drawn_and_bad_temperatures_rejected(oracle_mod):
    pen = np.array([[np.nan, -5.0, -6.0], [1.0, np.nan, 0.0]], np.float32)
    g = np.array([[0.0, 0.0, 0.5], [0.0, 0.0, np.nan]], np.float32)
    np.testing.assert_array_equal(oracle_mod.sample_targets(pen, g, 1.0), [1, 0])
    for bad in (0.0, -1.0, np.inf, np.nan):
        with pytest.raises(ValueError):
            oracle_mod.sample_targets(pen, g, bad)


def test_commit_golden_case(oracle_mod):
    c = json.load(open(SAMPLING))["commit"]
    cache = np.array(c["rows"], np.uint16)[None]
    out = oracle_mod.kv_commit_path(cache, c["n_ctx"], c["n_tree"], c["accept"])
    np.testing.assert_array_equal(out[0], np.array(c["expected_rows"], np.uint16))
    np.testing.assert_array_equal(cache[0], np.array(c["rows"], np.uint16))   # input untouched


def test_commit_moves_exactly_the_path_rows(oracle_mod):
    """Random caches and accepted paths: rows n_ctx + j hold the old rows of
    the path nodes, every other row is unchanged; L = 0 changes nothing."""
    rng = np.random.default_rng(24)
    for trial in range(30):
        hkv, d, n_ctx, t = 3, 8, int(rng.integers(0, 20)), int(rng.integers(1, 30))
        cap = n_ctx + t + int(rng.integers(0, 4))
        cache = rng.integers(0, 65535, size=(hkv, cap, d)).astype(np.uint16)
        parent = np.array([-1] + [int(rng.integers(0, i)) for i in range(1, t)], np.int32)
        end = int(rng.integers(0, t))
        path, a = [], end
        while a >= 0:
            path.append(a)
            a = int(parent[a])
        path.reverse()
        acc = np.array([len(path) - 1, 0] + path, np.int32)
        out = oracle_mod.kv_commit_path(cache, n_ctx, t, acc)
        want = cache.copy()
        for j, node in enumerate(path):
            want[:, n_ctx + j] = cache[:, n_ctx + node]
        np.testing.assert_array_equal(out, want)
    cache = rng.integers(0, 65535, size=(2, 10, 4)).astype(np.uint16)
    np.testing.assert_array_equal(oracle_mod.kv_commit_path(cache, 3, 5, [0, 1, 0]), cache)
