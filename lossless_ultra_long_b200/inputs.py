"""Seeded synthetic inputs for the TokenSwift verification path.

This module holds no arithmetic of the method itself: it draws random
numbers, rounds them to bf16 storage, and lays out the tree structures the
method consumes.  Both the fp64 CPU oracle (through the tests) and the CUDA
library are fed from here, so the two sides never see different inputs.

Recipe (all seeds are numpy PCG64 ``default_rng`` SeedSequences):

* Q, K, V: fp32 standard normal, rounded to bf16 with round-to-nearest-even.
  K and V are stored head-major ``[Hkv, kv_cap, D]``; rows ``[0, n_ctx)`` are
  the context, rows ``[n_ctx, n_ctx + T)`` the draft-tree tail.
* Key spikes (the 100K LLaMA-8B workload): ``floor(0.01 * n_ctx)`` distinct
  context positions in ``[n_sink, n_ctx)`` get +3.0 (three standard
  deviations) added to every element of K, for every KV head, before the
  bf16 rounding.
* Logits: fp32 normal with standard deviation 2.
* Penalty window: ids drawn uniformly from ``[0, V)`` with replacement.
* Gumbel noise (the temperature draw's randomness): ``-log(-log(u))`` with
  ``u`` uniform on ``[0, 1)`` in fp64 (a zero replaced by the smallest
  positive double), stored as fp32 ``[T, V]``.
* Tree: a 3-ary tree in BFS order, ``parent[i] = (i - 1) // 3``; a chain is
  ``parent[i] = i - 1``.
* Tree tokens: per node, with probability 0.7 one randomly chosen child gets
  a "planted" token id and that id's logit at the parent is raised to
  ``PLANT_LOGIT`` (far above any N(0, 2) draw, and still above it after a
  division by the penalty), so the greedy walk accepts a spread of lengths;
  every other child gets a random id different from the planted one.
"""
from __future__ import annotations

import dataclasses
import numpy as np

PLANT_LOGIT = 64.0


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(stream)])


# Per-tensor sub-streams so that any one tensor can be regenerated alone.
_S_Q, _S_K, _S_V, _S_LOGITS, _S_WINDOW, _S_TOKENS, _S_SPIKE, _S_DRAFTQ, _S_GUMBEL = range(1, 10)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bfs_tree(n_nodes: int, arity: int = 3) -> np.ndarray:
    """Parent array of a complete ``arity``-ary tree numbered in BFS order."""
    p = np.empty(n_nodes, dtype=np.int32)
    p[0] = -1
    for i in range(1, n_nodes):
        p[i] = (i - 1) // arity
    return p


def chain_tree(n_nodes: int) -> np.ndarray:
    p = np.arange(-1, n_nodes - 1, dtype=np.int32)
    return p


def ternary_nodes(depth: int) -> int:
    """Nodes of a full 3-ary tree of the given depth: 1 + 3 + ... + 3**depth."""
    return sum(3 ** d for d in range(depth + 1))


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n_heads_q: int
    n_heads_kv: int
    head_dim: int
    n_ctx: int
    n_tree: int
    tree: str = "ternary"          # "ternary" or "chain"
    vocab: int = 0
    window: int = 0
    penalty: float = 1.2
    n_sink: int = 0
    budget: int = 0
    spike: bool = False
    draft_tree: int = 0            # chain length of the draft pass over the partial cache
    seed: int = 0

    @property
    def group(self) -> int:
        return self.n_heads_q // self.n_heads_kv

    @property
    def kv_rows(self) -> int:
        return self.n_ctx + self.n_tree

    def parent(self) -> np.ndarray:
        return chain_tree(self.n_tree) if self.tree == "chain" else bfs_tree(self.n_tree)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads of the verification path.  Sizes follow the
# LLaMA3.1-8B / 7B-MHA / 14B-GQA attention shapes the TokenSwift pages name.
TINY = Workload("tiny_gqa8x2_d64_n2048_t13", 8, 2, 64, 2048, 13, vocab=4096, window=256,
                n_sink=16, budget=240, seed=0)
LLAMA8B_32K = Workload("llama8b_gqa32x8_d128_n32768_t40", 32, 8, 128, 32768, 40,
                       vocab=128256, window=1024, n_sink=64, budget=4032, seed=1)
LLAMA8B_100K = Workload("llama8b_gqa32x8_d128_n102400_t40", 32, 8, 128, 102400, 40,
                        vocab=128256, window=1024, n_sink=64, budget=4032, spike=True,
                        draft_tree=4, seed=2)
MHA7B_100K = Workload("mha7b_32x32_d128_n102400_t40", 32, 32, 128, 102400, 40,
                      vocab=32000, window=1024, n_sink=64, budget=4032, seed=3)
SWEEP_CTX = (4096, 16384, 65536, 102400, 131072)
SWEEP_TREE = (4, 13, 40)


def sweep14b(n_ctx: int, n_tree: int) -> Workload:
    return Workload(f"qwen14b_gqa40x8_d128_n{n_ctx}_t{n_tree}", 40, 8, 128, n_ctx, n_tree,
                    tree="chain" if n_tree == 4 else "ternary", seed=4)


ALL = {w.name: w for w in (TINY, LLAMA8B_32K, LLAMA8B_100K, MHA7B_100K)}


# ---------------------------------------------------------------- generators
def gen_q(w: Workload, n_nodes: int | None = None, stream: int = _S_Q) -> np.ndarray:
    """bf16 bits ``[T, Hq, D]``."""
    t = w.n_tree if n_nodes is None else n_nodes
    x = _rng(w.seed, stream).standard_normal((t, w.n_heads_q, w.head_dim), dtype=np.float32)
    return f32_to_bf16_bits(x)


def gen_draft_q(w: Workload) -> np.ndarray:
    return gen_q(w, w.draft_tree, stream=_S_DRAFTQ)


def spike_positions(w: Workload) -> np.ndarray:
    if not w.spike:
        return np.zeros(0, dtype=np.int64)
    n = int(0.01 * w.n_ctx)
    lo = w.n_sink
    pos = _rng(w.seed, _S_SPIKE).choice(w.n_ctx - lo, size=n, replace=False) + lo
    return np.sort(pos).astype(np.int64)


def gen_kv(w: Workload, kv_cap: int | None = None) -> tuple[np.ndarray, np.ndarray]:
    """bf16 bits K, V ``[Hkv, kv_cap, D]``; rows past n_ctx + T are zero."""
    cap = w.kv_rows if kv_cap is None else kv_cap
    assert cap >= w.kv_rows
    shape = (w.n_heads_kv, w.kv_rows, w.head_dim)
    out = []
    for stream in (_S_K, _S_V):
        x = _rng(w.seed, stream).standard_normal(shape, dtype=np.float32)
        if stream == _S_K and w.spike:
            x[:, spike_positions(w), :] += np.float32(3.0)
        b = f32_to_bf16_bits(x)
        if cap != w.kv_rows:
            full = np.zeros((w.n_heads_kv, cap, w.head_dim), dtype=np.uint16)
            full[:, : w.kv_rows] = b
            b = full
        out.append(b)
    return out[0], out[1]


def gen_logits(w: Workload) -> np.ndarray:
    """fp32 ``[T, V]`` with N(0, 2) entries (2 is the standard deviation)."""
    return _rng(w.seed, _S_LOGITS).normal(0.0, 2.0, size=(w.n_tree, w.vocab)).astype(np.float32)


def gen_gumbel(w: Workload, draw: int = 0) -> np.ndarray:
    """fp32 ``[T, V]`` standard Gumbel noise; ``draw`` selects an independent
    draw for the same workload."""
    u = _rng(w.seed * 1000 + draw, _S_GUMBEL).random(size=(w.n_tree, w.vocab))
    u[u == 0.0] = np.finfo(np.float64).tiny
    return (-np.log(-np.log(u))).astype(np.float32)


def gen_window(w: Workload) -> np.ndarray:
    return _rng(w.seed, _S_WINDOW).integers(0, w.vocab, size=w.window, dtype=np.int64).astype(np.int32)


def gen_tree_tokens(w: Workload, parent: np.ndarray, logits: np.ndarray,
                    p_plant: float = 0.7) -> tuple[np.ndarray, np.ndarray]:
    """Draft-tree token ids ``[T]`` and the logits with planted maxima.

    Returns ``(tokens, logits_planted)``; ``tokens[0]`` (the root, an already
    accepted token) is a random id.  ``logits`` is copied, not modified.
    """
    rng = _rng(w.seed, _S_TOKENS)
    t = len(parent)
    tokens = rng.integers(0, w.vocab, size=t, dtype=np.int64).astype(np.int32)
    lg = np.array(logits, dtype=np.float32, copy=True)
    children = [[] for _ in range(t)]
    for c in range(1, t):
        children[int(parent[c])].append(c)
    for node in range(t):
        kids = children[node]
        if not kids:
            continue
        if rng.random() < p_plant:
            planted = int(rng.integers(0, w.vocab))
            slot = kids[int(rng.integers(0, len(kids)))]
            lg[node, planted] = np.float32(PLANT_LOGIT)
            for c in kids:
                if c == slot:
                    tokens[c] = planted
                else:
                    while True:
                        r = int(rng.integers(0, w.vocab))
                        if r != planted:
                            break
                    tokens[c] = r
    return tokens, lg
