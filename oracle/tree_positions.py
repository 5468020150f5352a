"""Tree positions and rotary position embedding in fp64 — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this module; the CUDA path never does and shares no code with it.

What it computes:
- A speculated tree's node i sits ``depth(i)`` steps below the root, and the root is
  the token right after the L_b cached tokens, so its position is L_b + depth(i)
  (LongSpec, gist.science summary, section 2C: the tree tokens are the new tokens after
  the cached part; siblings are alternatives for one position).
- Rotary position embedding (RoFormer: Enhanced Transformer with Rotary Position
  Embedding, listed under "Builds on" on the mlsanity page: each two-dimensional pair
  is turned by the angle position * theta_e, theta_e = base^(-2e/d)). The pairs are (x[e], x[e + d/2]), the half-split order of the
  Llama and Qwen models that the pages evaluate (their reference code names the helper
  ``rotate_half``). Written here as a plain 2x2 rotation per pair in fp64.
- The rotated values are rounded to bf16 (round to nearest, ties to even), which is
  what a caller that rotates its own bf16 tensors would hand to the attention.

Depths are found by walking parent links to the root, one node at a time.
"""
from __future__ import annotations

import numpy as np


class BadTree(ValueError):
    pass


def tree_depth_walk(parent_local) -> np.ndarray:
    """Depth of every node of one tree (root = node 0, parent -1; parent[i] in [0, i))."""
    par = np.asarray(parent_local, dtype=np.int64)
    n = len(par)
    depth = np.zeros(n, dtype=np.int64)
    if n and par[0] != -1:
        raise BadTree("node 0 is not a root")
    for i in range(n):
        x, steps = i, 0
        while x != 0:
            p = int(par[x])
            if p < 0 or p >= x:
                raise BadTree(f"node {x} has parent {p}")
            x = p
            steps += 1
        depth[i] = steps
    return depth


def tree_positions(parent, cu_seqlens, node_offsets) -> np.ndarray:
    """Position L_b + depth(i) of every tree node of the batch, in packed node order."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    off = np.asarray(node_offsets, dtype=np.int64)
    pos = np.zeros(int(off[-1]), dtype=np.int64)
    for b in range(len(off) - 1):
        s, e = int(off[b]), int(off[b + 1])
        if e > s:
            pos[s:e] = (cu[b + 1] - cu[b]) + tree_depth_walk(parent[s:e])
    return pos


def rope_rotate(x, positions, theta: float) -> np.ndarray:
    """Rotate fp64 x [n, H, d] for positions [n]: pair (x[e], x[e+d/2]) by pos * theta_e."""
    x = np.asarray(x, dtype=np.float64)
    n, H, d = x.shape
    half = d // 2
    e = np.arange(half, dtype=np.float64)
    theta_e = np.power(float(theta), -2.0 * e / d)                 # [half]
    ang = np.asarray(positions, dtype=np.float64)[:, None] * theta_e[None, :]  # [n, half]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    out = np.empty_like(x)
    out[..., :half] = x1 * c - x2 * s
    out[..., half:] = x2 * c + x1 * s
    return out


def round_to_bf16(x) -> np.ndarray:
    """fp64 -> nearest bf16 value (8 significant bits, ties to even), returned as fp64.
    Normal range only (the tests' values are far from bf16's limits)."""
    x = np.asarray(x, dtype=np.float64)
    m, ex = np.frexp(x)                      # x = m * 2^ex, 0.5 <= |m| < 1
    return np.ldexp(np.rint(np.ldexp(m, 8)), ex - 8)


def bf16_bits(x_bf16_valued) -> np.ndarray:
    """bf16-representable fp64 values -> uint16 bit patterns (exact)."""
    f = np.ascontiguousarray(np.asarray(x_bf16_valued, dtype=np.float64).astype(np.float32))
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bits_to_f64(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def rope_bf16(bits, positions, theta: float) -> np.ndarray:
    """bf16 bits [n, H, d] -> RoPE-rotated values rounded to bf16, as bits."""
    return bf16_bits(round_to_bf16(rope_rotate(bits_to_f64(bits), positions, theta)))


__all__ = ["BadTree", "tree_depth_walk", "tree_positions", "rope_rotate", "round_to_bf16", "bf16_bits",
           "bits_to_f64", "rope_bf16"]
