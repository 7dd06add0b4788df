"""The n-gram reuse table: the oracle against hand-worked and closed-form
counts, then the library's table (host code, ts_ngram_*) against the
oracle, exactly."""
import json
import os

import numpy as np
import pytest

from oracle import ngram as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "ngram_figure.json")


# ------------------------------------------------------------ oracle pins
def test_oracle_hand_counted_alternation():
    # 0 1 0 1 0: bigrams 01 at 0, 2 and 10 at 1, 3; trigrams 010 at 0, 2 and 101 at 1
    assert O.ngram_counts([0, 1, 0, 1, 0], 2) == {(0, 1): 2, (1, 0): 2}
    assert O.ngram_counts([0, 1, 0, 1, 0], 3) == {(0, 1, 0): 2, (1, 0, 1): 1}
    assert O.ngram_counts([0, 1, 0, 1, 0], 6) == {}


@pytest.mark.parametrize("p,length,n", [(3, 20, 2), (5, 31, 4), (7, 7, 7), (4, 100, 8)])
def test_oracle_periodic_text_closed_form(p, length, n):
    # text[i] = i mod p: the window starting at i is fixed by r = i mod p, and
    # the starts i in [0, length - n] with i = r (mod p) number
    # floor((length - n - r) / p) + 1
    text = [i % p for i in range(length)]
    got = O.ngram_counts(text, n)
    want = {}
    for r in range(min(p, length - n + 1)):
        g = tuple((r + j) % p for j in range(n))
        want[g] = (length - n - r) // p + 1
    assert got == want
    assert sum(got.values()) == length - n + 1


def test_oracle_distinct_tokens_count_once():
    got = O.ngram_counts(list(range(50)), 4)
    assert len(got) == 47 and set(got.values()) == {1}


def test_oracle_golden_figure_example():
    g = json.load(open(GOLDEN))
    ids = {w: i for i, w in enumerate(g["vocab"])}
    enc = lambda ws: [ids[w] for w in ws]
    n = g["n"]
    text = enc(g["text"])
    c = O.ngram_counts(text, n)
    assert sum(c.values()) == g["windows"]
    want = [(tuple(enc(cont)), cnt) for cont, cnt in g["topk_is"]]
    assert O.ngram_topk(c, ids["is"], 3) == want
    text2 = text + enc(g["appended"])
    c2 = O.ngram_update(c, text2, len(g["appended"]), n)
    assert sum(c2.values()) == g["windows_after"]
    diff = {k: c2[k] - c.get(k, 0) for k in c2 if c2[k] != c.get(k, 0)}
    assert diff == {tuple(enc(w)): 1 for w in g["new_windows"]}
    want2 = [(tuple(enc(cont)), cnt) for cont, cnt in g["topk_is_after"]]
    assert O.ngram_topk(c2, ids["is"], 3) == want2
    pre = enc(["is", "the", "uncle"])
    for cc, key in ((c, "next_after_is_the_uncle"), (c2, "next_after_is_the_uncle_after")):
        assert O.ngram_topk_prefix(cc, pre, 5) == [(tuple(enc(t)), k) for t, k in g[key]]


def test_oracle_update_counts_only_windows_ending_in_the_new_tokens():
    rng = np.random.default_rng(7)
    text = rng.integers(0, 4, 200).tolist()
    for n in (2, 3, 5):
        c, prev = O.ngram_counts(text[:120], n), 120
        for cut in (121, 150, 200):
            c = O.ngram_update(c, text[:cut], cut - prev, n)
            prev = cut
            assert c == O.ngram_counts(text[:cut], n)


def test_oracle_topk_order_breaks_ties_by_continuation():
    c = {(1, 5, 5): 2, (1, 2, 9): 2, (1, 2, 3): 2, (1, 0, 0): 1, (2, 0, 0): 9}
    assert O.ngram_topk(c, 1, 10) == [((2, 3), 2), ((2, 9), 2), ((5, 5), 2), ((0, 0), 1)]
    assert O.ngram_topk(c, 1, 2) == [((2, 3), 2), ((2, 9), 2)]
    assert O.ngram_topk(c, 3, 4) == []
    # a two-token prefix keeps only the n-grams that start with both tokens
    assert O.ngram_topk_prefix(c, [1, 2], 10) == [((3,), 2), ((9,), 2)]
    assert O.ngram_topk_prefix(c, [1], 10) == O.ngram_topk(c, 1, 10)
    assert O.ngram_topk_prefix(c, [2, 1], 10) == []


# ------------------------------------------------- the library's table
@pytest.fixture(scope="module")
def L():
    from lossless_ultra_long_b200 import build
    build.build()
    import lossless_ultra_long_b200 as L
    return L


def _rows(cont, cnt):
    return [(tuple(r), int(x)) for r, x in zip(cont.tolist(), cnt.tolist())]


def _same_as_oracle(tab, counts, n, firsts, ks=(1, 3, 16, 17, 50), n_prefixes=12):
    assert tab.size() == (len(counts), sum(counts.values()))
    for g, c in counts.items():
        assert tab.count(g) == c
    for first in firsts:
        for k in ks:
            assert _rows(*tab.topk(first, k)) == O.ngram_topk(counts, first, k)
    # every prefix length, on prefixes that occur and one that does not
    grams = sorted(counts)
    for p in range(1, n):
        picks = [grams[i][:p] for i in range(0, len(grams), max(1, len(grams) // n_prefixes))]
        picks.append((10 ** 6,) * p)
        for pre in picks:
            for k in ks:
                assert _rows(*tab.topk_prefix(pre, k)) == O.ngram_topk_prefix(counts, pre, k)


@pytest.mark.parametrize("n,vocab,length,seed", [(2, 3, 400, 0), (3, 5, 1000, 1), (4, 8, 3000, 2),
                                                 (8, 2, 600, 3), (4, 1000, 2000, 4)])
def test_table_matches_oracle_under_chunked_updates(L, n, vocab, length, seed):
    rng = np.random.default_rng(seed)
    text = rng.integers(0, vocab, length).astype(np.int32)
    tab = L.NgramTable(n, 1 << 13)
    counts, done = {}, 0
    while done < length:
        step = int(rng.integers(1, 60))
        cut = min(length, done + step)
        # pass only the tail the new windows need, as a generator would
        lo = max(0, done - (n - 1))
        tab.update(text[lo:cut], cut - done)
        counts = O.ngram_update(counts, text[:cut].tolist(), cut - done, n)
        done = cut
    assert counts == O.ngram_counts(text.tolist(), n)
    _same_as_oracle(tab, counts, n, firsts=range(min(vocab, 12)))
    # absent n-grams and first tokens
    assert tab.count([vocab + 1] * n) == 0
    assert tab.topk(vocab + 5, 4)[1].size == 0


def test_table_golden_figure_example(L):
    g = json.load(open(GOLDEN))
    ids = {w: i for i, w in enumerate(g["vocab"])}
    enc = lambda ws: [ids[w] for w in ws]
    tab = L.NgramTable(g["n"], 64)
    text = enc(g["text"])
    tab.update(text)
    cont, cnt = tab.topk(ids["is"], 3)
    assert [(r, int(x)) for r, x in zip(cont.tolist(), cnt.tolist())] == \
        [(enc(c), k) for c, k in g["topk_is"]]
    tab.update(text + enc(g["appended"]), len(g["appended"]))
    assert tab.size()[1] == g["windows_after"]
    cont, cnt = tab.topk(ids["is"], 3)
    assert [(r, int(x)) for r, x in zip(cont.tolist(), cnt.tolist())] == \
        [(enc(c), k) for c, k in g["topk_is_after"]]
    cont, cnt = tab.topk_prefix(enc(["is", "the", "uncle"]), 4)
    assert [(r, int(x)) for r, x in zip(cont.tolist(), cnt.tolist())] == \
        [(enc(c), k) for c, k in g["next_after_is_the_uncle_after"]]


def test_table_full_is_all_or_nothing(L):
    # capacity 16 holds at most 14 distinct n-grams
    tab = L.NgramTable(2, 16)
    tab.update(list(range(15)))                   # 14 distinct bigrams: exactly full
    assert tab.size() == (14, 14)
    before = {(i, i + 1): 1 for i in range(14)}
    with pytest.raises(L.TsError) as e:
        tab.update([14, 15, 16], 2)               # two new bigrams
    assert e.value.status == 3
    assert tab.size() == (14, 14)
    for g, c in before.items():
        assert tab.count(g) == c
    tab.update([3, 4, 5, 6], 3)                   # only known bigrams: still fits
    assert tab.size() == (14, 17)
    assert tab.count((4, 5)) == 2


def test_table_short_texts_and_empty_updates(L):
    tab = L.NgramTable(4, 32)
    tab.update([1, 2, 3])                         # shorter than n: nothing to count
    tab.update([], 0)
    tab.update([1, 2, 3, 4], 0)                   # no new tokens
    assert tab.size() == (0, 0)
    tab.update([1, 2, 3, 4], 1)
    assert tab.size() == (1, 1) and tab.count([1, 2, 3, 4]) == 1


def test_table_rejects_invalid_calls(L):
    lib = L.library()
    assert lib.ts_ngram_table_bytes(1, 16) == 0
    assert lib.ts_ngram_table_bytes(9, 16) == 0
    assert lib.ts_ngram_table_bytes(4, 24) == 0          # not a power of two
    assert lib.ts_ngram_table_bytes(4, 16) == 64 + 16 * 216
    assert lib.ts_ngram_table_bytes(4, 1 << 32) == 0     # slot indices are int32
    with pytest.raises(ValueError):
        L.NgramTable(4, 12)
    tab = L.NgramTable(3, 16)
    with pytest.raises(L.TsError) as e:
        tab.update([1, -2, 3, 4], 1)                      # negative token in the window
    assert e.value.status == 1
    with pytest.raises(L.TsError):
        tab.update([1, 2, 3], 4)                          # more new tokens than text
    with pytest.raises(L.TsError):
        tab.topk(1, 0)
    with pytest.raises(L.TsError):
        tab.topk(1, 4097)
    with pytest.raises(L.TsError):
        tab.topk_prefix([1, 2, 3], 4)                     # prefix as long as n
    with pytest.raises(L.TsError):
        tab.topk_prefix([], 4)
    # an unformatted buffer is not a table
    import ctypes
    buf = np.zeros(200, dtype=np.uint64)
    c = ctypes.c_int64(0)
    gram = np.zeros(3, dtype=np.int32)
    assert lib.ts_ngram_count(buf.ctypes.data_as(ctypes.c_void_p), buf.nbytes,
                              gram.ctypes.data_as(ctypes.c_void_p), ctypes.byref(c)) == 1
    # a table_bytes smaller than the table it holds
    assert lib.ts_ngram_count(tab._p, tab.nbytes - 8, gram.ctypes.data_as(ctypes.c_void_p),
                              ctypes.byref(c)) == 1


def test_table_best_lists_stay_exact_as_counts_grow(L):
    # 3 tokens, n = 5: up to 81 continuations per first token, so the best
    # 16 are displaced over and over as the counts grow; checked after
    # every update against the oracle's order
    rng = np.random.default_rng(11)
    n = 5
    # a drifting distribution: which continuations lead changes over time
    text = np.concatenate([rng.choice(3, 700, p=p) for p in
                           ([0.6, 0.3, 0.1], [0.2, 0.2, 0.6], [0.34, 0.33, 0.33],
                            [0.1, 0.8, 0.1])]).astype(np.int32)
    tab = L.NgramTable(n, 1 << 10)
    counts, done = {}, 0
    while done < len(text):
        cut = min(len(text), done + int(rng.integers(1, 40)))
        tab.update(text[max(0, done - n + 1):cut], cut - done)
        counts = O.ngram_update(counts, text[:cut].tolist(), cut - done, n)
        done = cut
        for first in range(3):
            for k in (1, 5, 16):
                cont, cnt = tab.topk(first, k)
                assert [(tuple(r), int(x)) for r, x in zip(cont.tolist(), cnt.tolist())] == \
                    O.ngram_topk(counts, first, k)
    _same_as_oracle(tab, counts, n, firsts=range(3), ks=(16, 17, 81, 200))


def test_table_next_token_lists_stay_exact_as_counts_grow(L):
    # n = 3 over 40 tokens with a drifting skew: the frequent two-token
    # prefixes gather far more than 16 next tokens, so their best lists (the
    # second index) are displaced over and over; checked after every update
    rng = np.random.default_rng(12)
    n, vocab = 3, 40
    parts = []
    for shift in (0, 13, 27, 5):
        w = 1.0 / (1.0 + ((np.arange(vocab) + shift) % vocab))
        parts.append(rng.choice(vocab, 1500, p=w / w.sum()))
    text = np.concatenate(parts).astype(np.int32)
    tab = L.NgramTable(n, 1 << 14)
    counts, done = {}, 0
    watch = [(0, 0), (0, 1), (13, 13), (27, 27), (5, 5)]
    while done < len(text):
        cut = min(len(text), done + int(rng.integers(1, 50)))
        tab.update(text[max(0, done - n + 1):cut], cut - done)
        counts = O.ngram_update(counts, text[:cut].tolist(), cut - done, n)
        done = cut
        for pre in watch:
            for k in (1, 5, 16):
                assert _rows(*tab.topk_prefix(pre, k)) == O.ngram_topk_prefix(counts, pre, k)
    assert max(len(O.ngram_topk_prefix(counts, pre, 100)) for pre in watch) > 16
    _same_as_oracle(tab, counts, n, firsts=range(0, vocab, 3), ks=(16, 17, 40))
