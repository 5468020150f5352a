"""Seeded synthetic inputs for tree-verification attention.

This module only draws random numbers and builds tree shapes. It holds none of the
attention arithmetic, so both the fp64 oracle and the CUDA path can take their
inputs from here without sharing any of the method.

Every tensor is returned as raw bf16 bit patterns (``uint16``) so the two sides see
identical inputs. Floats are drawn as float32 from numpy's PCG64 and rounded to
bf16 with round-to-nearest-even.

Layouts (row-major, matching the C-ABI; N = B*T tree nodes, or cu_tree[B] when the
trees differ in size per sequence):
  q        [N, H_q, d]        tree queries, token-major
  k_cache  [sum L_b, H_kv, d] prefix keys, sequences packed by cu_seqlens
  v_cache  [sum L_b, H_kv, d]
  k_tree   [N, H_kv, d]       tree keys
  v_tree   [N, H_kv, d]
  parent   [N] int32          local parent index, -1 for the root (node 0)
  cu_seqlens [B+1] int32      prefix offsets, cu[0] = 0
  cu_tree  [B+1] int32        tree node offsets (per-sequence trees only), cu_tree[0] = 0

The tree shapes follow the verification setting of the LongSpec paper ("Hybrid
Tree Attention", gist.science summary, section 2C): a draft token tree whose
nodes are numbered so that every parent precedes its children.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np


# ----------------------------------------------------------------------------- bf16
def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 exactly."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(bits).astype(np.float64)


# ----------------------------------------------------------------------------- trees
def chain_tree(T: int) -> np.ndarray:
    """parent[i] = i - 1: a single speculated path (the tree degenerates to a sequence)."""
    p = np.arange(-1, T - 1, dtype=np.int32)
    return p


def star_tree(T: int) -> np.ndarray:
    """Every node hangs off the root."""
    p = np.zeros(T, dtype=np.int32)
    p[0] = -1
    return p


def window_tree(rng: np.random.Generator, T: int, window: Optional[int]) -> np.ndarray:
    """parent[i] ~ U[max(0, i - window), i) for i >= 1 (window=None: U[0, i))."""
    p = np.empty(T, dtype=np.int32)
    if T == 0:
        return p
    p[0] = -1
    for i in range(1, T):
        lo = 0 if window is None else max(0, i - window)
        p[i] = rng.integers(lo, i)
    return p


def bfs_tree(rng: np.random.Generator, T: int, max_children: int = 4,
             max_depth: int = 12) -> np.ndarray:
    if T == 0:
        return np.empty(0, dtype=np.int32)
    return _bfs_tree(rng, T, max_children, max_depth)


def _bfs_tree(rng: np.random.Generator, T: int, max_children: int, max_depth: int) -> np.ndarray:
    """Breadth-first tree: each dequeued node gets c ~ U{1..max_children} children,
    clipped to the nodes left and to depth <= max_depth (root depth 0). Nodes are
    numbered in BFS order, so parent[i] < i. If the frontier dies out before T nodes
    exist (every open node sits at max_depth), the draw is repeated from the same
    stream."""
    while True:
        p = np.full(T, -1, dtype=np.int32)
        depth = np.zeros(T, dtype=np.int32)
        queue = [0]
        n = 1
        head = 0
        while n < T and head < len(queue):
            node = queue[head]
            head += 1
            if depth[node] >= max_depth:
                continue
            c = int(rng.integers(1, max_children + 1))
            c = min(c, T - n)
            for _ in range(c):
                p[n] = node
                depth[n] = depth[node] + 1
                queue.append(n)
                n += 1
        if n == T:
            return p


def tree_depths(parent: np.ndarray) -> np.ndarray:
    """Depth of every node of one tree (root depth 0); parent[i] < i is assumed."""
    d = np.zeros(len(parent), dtype=np.int32)
    for i in range(1, len(parent)):
        d[i] = d[parent[i]] + 1
    return d


# ----------------------------------------------------------------------------- workloads
@dataclass(frozen=True)
class Workload:
    """One synthetic verification call.

    prefix: a fixed L for every sequence, or (lo, hi) for L_b ~ U{lo..hi} i.i.d.
    tree:   'uniform' (parent ~ U[0,i)), 'window8' (parent ~ U[max(0,i-8),i)),
            'bfs' (branching 1..4, depth <= 12), 'chain' or 'star'.
    input_scale: multiplier applied to the N(0,1) draws before bf16 rounding.
    tree_sizes / tree_size_range: per-sequence trees, T_b given or T_b ~ U{lo..hi} i.i.d.
            (tree_size is then the largest tree allowed); neither: T nodes each.
    """
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    tree_size: int
    prefix: object
    tree: str
    input_scale: float = 1.0
    lengths: Optional[Sequence[int]] = field(default=None)  # explicit L_b, overrides prefix
    tree_sizes: Optional[Sequence[int]] = field(default=None)
    tree_size_range: Optional[tuple] = field(default=None)

    @property
    def ragged_trees(self) -> bool:
        return self.tree_sizes is not None or self.tree_size_range is not None

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


def draw_prefix_lengths(w: Workload, rng: np.random.Generator) -> np.ndarray:
    if w.lengths is not None:
        L = np.asarray(w.lengths, dtype=np.int64)
        assert L.shape == (w.batch,)
        return L
    if isinstance(w.prefix, tuple):
        lo, hi = w.prefix
        return rng.integers(lo, hi + 1, size=w.batch).astype(np.int64)
    return np.full(w.batch, int(w.prefix), dtype=np.int64)


def draw_tree_sizes(w: Workload, rng: np.random.Generator) -> Optional[np.ndarray]:
    """T_b per sequence for per-sequence trees, else None (every tree has tree_size nodes)."""
    if w.tree_sizes is not None:
        t = np.asarray(w.tree_sizes, dtype=np.int64)
        assert t.shape == (w.batch,) and t.min() >= 0 and t.max() <= w.tree_size
        return t
    if w.tree_size_range is not None:
        lo, hi = w.tree_size_range
        assert 0 <= lo <= hi <= w.tree_size
        return rng.integers(lo, hi + 1, size=w.batch).astype(np.int64)
    return None


def draw_tree(kind: str, rng: np.random.Generator, T: int) -> np.ndarray:
    if kind == "uniform":
        return window_tree(rng, T, None)
    if kind == "window8":
        return window_tree(rng, T, 8)
    if kind == "bfs":
        return bfs_tree(rng, T)
    if kind == "chain":
        return chain_tree(T)
    if kind == "star":
        return star_tree(T)
    raise ValueError(f"unknown tree kind {kind!r}")


@dataclass
class Inputs:
    workload: Workload
    q: np.ndarray
    k_cache: np.ndarray
    v_cache: np.ndarray
    k_tree: np.ndarray
    v_tree: np.ndarray
    parent: np.ndarray
    cu_seqlens: np.ndarray
    seed: int
    cu_tree: Optional[np.ndarray] = None  # per-sequence trees: node offsets [B+1]

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.workload.head_dim))

    @property
    def prefix_lengths(self) -> np.ndarray:
        return np.diff(self.cu_seqlens).astype(np.int64)

    @property
    def num_nodes(self) -> int:
        return int(self.q.shape[0])

    def node_offsets(self) -> np.ndarray:
        """cu_tree, or b * T for uniform trees."""
        if self.cu_tree is not None:
            return self.cu_tree
        w = self.workload
        return (np.arange(w.batch + 1) * w.tree_size).astype(np.int32)


def _normal_bf16(rng: np.random.Generator, shape, scale: float) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return bf16_bits_from_f32(x)


def make_inputs(w: Workload, seed: int = 0) -> Inputs:
    """Draw the inputs of workload ``w``.

    Structure (prefix lengths, per-sequence tree sizes when the workload has them, then
    one tree per sequence) comes from ``default_rng(seed + 1)``; tensors come from
    ``default_rng(seed)`` in the order q, k_cache, v_cache, k_tree, v_tree.
    """
    srng = np.random.default_rng(seed + 1)
    L = draw_prefix_lengths(w, srng)
    sizes = draw_tree_sizes(w, srng)
    tb = sizes if sizes is not None else np.full(w.batch, w.tree_size, dtype=np.int64)
    parents = [draw_tree(w.tree, srng, int(t)) for t in tb]
    parent = np.concatenate(parents).astype(np.int32)
    cu = np.zeros(w.batch + 1, dtype=np.int32)
    cu[1:] = np.cumsum(L)
    total_L = int(cu[-1])
    cu_tree = None
    if sizes is not None:
        cu_tree = np.zeros(w.batch + 1, dtype=np.int32)
        cu_tree[1:] = np.cumsum(sizes)
    N = int(tb.sum())

    trng = np.random.default_rng(seed)
    Hq, Hkv, d = w.num_q_heads, w.num_kv_heads, w.head_dim
    s = w.input_scale
    q = _normal_bf16(trng, (N, Hq, d), s)
    k_cache = _normal_bf16(trng, (total_L, Hkv, d), s)
    v_cache = _normal_bf16(trng, (total_L, Hkv, d), s)
    k_tree = _normal_bf16(trng, (N, Hkv, d), s)
    v_tree = _normal_bf16(trng, (N, Hkv, d), s)
    return Inputs(w, q, k_cache, v_cache, k_tree, v_tree, parent, cu, seed, cu_tree)


# ----------------------------------------------------------------------------- acceptance
@dataclass
class AcceptInputs:
    """One greedy-acceptance step: logits of every tree node, draft tokens, tree."""
    logits: np.ndarray            # [N, V] bf16 bits (uint16) or float32
    tokens: np.ndarray            # [N] int32 draft tokens (node 0's unused)
    parent: np.ndarray            # [N] int32 local parents
    cu_tree: Optional[np.ndarray]  # [B+1] int32, or None (T nodes each)
    batch: int
    tree_size: int
    vocab: int
    dtype: str                    # "bf16" or "f32"


def make_accept_inputs(batch: int, tree_size: int, vocab: int, dtype: str = "bf16", tree: str = "window8",
                       match_prob: float = 0.7, seed: int = 0,
                       tree_sizes: Optional[Sequence[int]] = None) -> AcceptInputs:
    """Logits N(0,1) with one planted peak per node (value 8 at a random token), and draft
    tokens that copy the parent's planted token with probability match_prob (else a
    random token), so that walks of several steps occur. Nothing here computes an
    argmax: the planted peak is only where the generator put the large value.
    Structure from ``default_rng(seed + 1)``, values from ``default_rng(seed)``."""
    srng = np.random.default_rng(seed + 1)
    sizes = (np.full(batch, tree_size, dtype=np.int64) if tree_sizes is None
             else np.asarray(tree_sizes, dtype=np.int64))
    parents = [draw_tree(tree, srng, int(t)) for t in sizes]
    parent = np.concatenate(parents).astype(np.int32) if len(parents) else np.zeros(0, np.int32)
    N = int(sizes.sum())
    cu_tree = None
    if tree_sizes is not None:
        cu_tree = np.zeros(batch + 1, dtype=np.int32)
        cu_tree[1:] = np.cumsum(sizes)
    vrng = np.random.default_rng(seed)
    x = vrng.standard_normal(size=(N, vocab), dtype=np.float32)
    peak = vrng.integers(0, vocab, size=N)
    x[np.arange(N), peak] = 8.0
    tokens = vrng.integers(0, vocab, size=N).astype(np.int32)
    copy = vrng.random(N) < match_prob
    off = 0
    for t in sizes:
        for i in range(1, int(t)):
            if copy[off + i]:
                tokens[off + i] = peak[off + parent[off + i]]
        off += int(t)
    logits = bf16_bits_from_f32(x) if dtype == "bf16" else x
    return AcceptInputs(logits, tokens, parent, cu_tree, batch, tree_size, vocab, dtype)
