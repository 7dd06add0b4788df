"""Plain n-gram counting for the n-gram reuse table.

TEST INFRASTRUCTURE ONLY (tests and the smoke check); never imported by the
product library.  Pure Python over small token lists: a dictionary from
each run of n consecutive tokens to its number of occurrences.

Source: TokenSwift reuses phrases that recur in the generated text, by
their n-gram frequencies, as draft candidates, and updates the n-gram table
after each verification ("TokenSwift - A framework for accelerating the
generation of ultra-long text", aiboss88.com, "Parallel generation of
multiple tokens and token reuse"; cloud.tencent.com article, the
parallel-verification step of the method figure).  The pages fix neither n
nor the retrieval order; the reading taken here: count every window of n
tokens; the candidates for a prefix (a first token, or the last n-1
tokens) are the n-grams that start with it, by count, descending, ties by
continuation in ascending token order.
"""
from __future__ import annotations


def ngram_counts(text, n):
    """Occurrences of every window text[i:i+n], i = 0 .. len(text) - n."""
    counts = {}
    for i in range(len(text) - n + 1):
        g = tuple(int(x) for x in text[i:i + n])
        counts[g] = counts.get(g, 0) + 1
    return counts


def ngram_update(counts, text, n_new, n):
    """The counts after the last n_new tokens of `text` were generated: every
    window that ends at one of those positions is counted once more."""
    out = dict(counts)
    for e in range(max(n - 1, len(text) - n_new), len(text)):
        g = tuple(int(x) for x in text[e - n + 1:e + 1])
        out[g] = out.get(g, 0) + 1
    return out


def ngram_topk(counts, first, k):
    """The k most frequent n-grams that start with `first`, as
    (continuation, count) pairs: count descending, then continuation
    ascending."""
    cands = [(g[1:], c) for g, c in counts.items() if g[0] == first]
    cands.sort(key=lambda gc: (-gc[1], gc[0]))
    return cands[:k]


def ngram_topk_prefix(counts, prefix, k):
    """The k most frequent n-grams that start with the tokens of `prefix`,
    as (continuation, count) pairs in the same order as ngram_topk."""
    p = len(prefix)
    pre = tuple(int(x) for x in prefix)
    cands = [(g[p:], c) for g, c in counts.items() if g[:p] == pre]
    cands.sort(key=lambda gc: (-gc[1], gc[0]))
    return cands[:k]
