"""fp64 CPU oracle for tree-verification attention — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA product path never does, and the
two share no code; they meet only at the seeded inputs.

``verify_attn_oracle`` is one softmax over prefix U ancestors-or-self per query
row (LongSpec, gist.science summary, section 2C), computed in fp64 from the exact
bf16 inputs by ``verify_attn_oracle.c``. ``softmax_keyset`` is the same softmax over
an explicit key list, used by the tests to check the log-sum-exp merge.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        lib.oracle_verify_attn.argtypes = [P, P, P, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_double, P, ctypes.c_int64, P, P,
                                           ctypes.c_int]
        lib.oracle_verify_attn.restype = ctypes.c_int
        lib.oracle_softmax_keyset.argtypes = [P, P, P, ctypes.c_int64, ctypes.c_int64,
                                              ctypes.c_int, ctypes.c_double, P, P]
        lib.oracle_softmax_keyset.restype = None
        lib.oracle_check_trees.argtypes = [P, ctypes.c_int, ctypes.c_int]
        lib.oracle_check_trees.restype = ctypes.c_int
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def verify_attn_oracle(q, k_cache, v_cache, k_tree, v_tree, parent, cu_seqlens,
                       *, num_q_heads: int, num_kv_heads: int, head_dim: int, tree_size: int,
                       scale: Optional[float] = None, rows: Optional[np.ndarray] = None,
                       nthreads: int = 0):
    """Returns (out fp64 [n, d], lse fp64 [n]) for the selected rows.

    Row r = (b*T + i)*H_q + h. rows=None computes all B*T*H_q rows in that order.
    Tensors are bf16 bit patterns (uint16) in the C-ABI layouts.
    """
    lib = _load()
    d, T = head_dim, tree_size
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    B = len(cu) - 1
    if scale is None:
        scale = 1.0 / float(np.sqrt(d))
    arrs = [np.ascontiguousarray(a, dtype=np.uint16) for a in (q, k_cache, v_cache, k_tree, v_tree)]
    par = np.ascontiguousarray(parent, dtype=np.int32)
    if rows is None:
        n = B * T * num_q_heads
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n = len(rows_arr)
    out = np.empty((n, d), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    rc = lib.oracle_verify_attn(*[_ptr(a) for a in arrs], _ptr(par), _ptr(cu), B, num_q_heads,
                                num_kv_heads, d, T, float(scale),
                                None if rows_arr is None else _ptr(rows_arr), n,
                                _ptr(out), _ptr(lse), int(nthreads))
    if rc != 0:
        raise OracleError({1: "bad argument", 2: "bad tree", 3: "out of memory"}.get(rc, rc))
    return out, lse


def verify_attn_oracle_inputs(inp, rows=None, nthreads: int = 0, scale=None):
    """Convenience: run the oracle on an ``inputs.Inputs`` bundle."""
    w = inp.workload
    return verify_attn_oracle(inp.q, inp.k_cache, inp.v_cache, inp.k_tree, inp.v_tree,
                              inp.parent, inp.cu_seqlens, num_q_heads=w.num_q_heads,
                              num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                              tree_size=w.tree_size, scale=scale if scale is not None else inp.scale,
                              rows=rows, nthreads=nthreads)


def verify_attn_oracle_packed(q, k_cache, v_cache, k_tree, v_tree, parent, cu_seqlens, node_offsets,
                              *, num_q_heads: int, num_kv_heads: int, head_dim: int, scale: float,
                              nthreads: int = 0):
    """Trees of different sizes: sequence b's nodes are rows [off[b], off[b+1]) of q,
    k_tree, v_tree and parent. Each sequence is its own one-sequence problem with
    T_b = off[b+1] - off[b] nodes. Returns (out [N*H_q, d], lse [N*H_q]) in packed
    row order (node n, head h) -> n*H_q + h."""
    off = np.asarray(node_offsets, dtype=np.int64)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    N = int(off[-1])
    out = np.zeros((N * num_q_heads, head_dim))
    lse = np.zeros(N * num_q_heads)
    for b in range(len(off) - 1):
        s, e = int(off[b]), int(off[b + 1])
        if e == s:
            continue
        l0, l1 = int(cu[b]), int(cu[b + 1])
        o, l_ = verify_attn_oracle(q[s:e], k_cache[l0:l1], v_cache[l0:l1], k_tree[s:e], v_tree[s:e],
                                   parent[s:e], np.array([0, l1 - l0], dtype=np.int32),
                                   num_q_heads=num_q_heads, num_kv_heads=num_kv_heads, head_dim=head_dim,
                                   tree_size=e - s, scale=scale, nthreads=nthreads)
        out[s * num_q_heads:e * num_q_heads] = o
        lse[s * num_q_heads:e * num_q_heads] = l_
    return out, lse


def verify_attn_oracle_window(q, k_cache, v_cache, k_tree, v_tree, parent, cu_seqlens, node_offsets, *,
                              num_q_heads: int, num_kv_heads: int, head_dim: int, scale: float, window: int,
                              rows=None):
    """Sliding-window attention (LongSpec, gist.science summary, section 2A): a query at
    position P sees the keys at positions P - window + 1 .. P. Prefix key j of sequence b
    sits at position j and tree node i at L_b + depth(i), so row (node i, head h) attends
    the prefix keys j >= L_b + depth(i) + 1 - window and the tree nodes a on its root path
    with depth(i) - depth(a) < window. Each row is one fp64 softmax over that explicit key
    list (``softmax_keyset``). Rows are packed (node n, head h) -> n*H_q + h; rows=None
    computes all of them. Returns (out [n, d], lse [n])."""
    from .tree_positions import tree_depth_walk
    off = np.asarray(node_offsets, dtype=np.int64)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    g = num_q_heads // num_kv_heads
    N = int(off[-1])
    rows = np.arange(N * num_q_heads) if rows is None else np.asarray(rows, dtype=np.int64)
    seq_of = np.searchsorted(off, np.arange(N), side="right") - 1
    depth = np.zeros(N, dtype=np.int64)
    for b in range(len(off) - 1):
        if off[b + 1] > off[b]:
            depth[off[b]:off[b + 1]] = tree_depth_walk(parent[off[b]:off[b + 1]])
    out = np.zeros((len(rows), head_dim))
    lse = np.zeros(len(rows))
    for r_i, r in enumerate(rows):
        n, h = divmod(int(r), num_q_heads)
        b = int(seq_of[n])
        i = n - int(off[b])
        kh = h // g
        L = int(cu[b + 1] - cu[b])
        j0 = max(0, L + int(depth[n]) + 1 - window)
        path = []
        x = i
        while True:
            if int(depth[n]) - int(depth[int(off[b]) + x]) < window:
                path.append(int(off[b]) + x)
            if x == 0:
                break
            x = int(parent[int(off[b]) + x])
        keys = np.concatenate([k_cache[int(cu[b]) + j0:int(cu[b + 1]), kh], k_tree[path, kh]])
        vals = np.concatenate([v_cache[int(cu[b]) + j0:int(cu[b + 1]), kh], v_tree[path, kh]])
        out[r_i], lse[r_i] = softmax_keyset(q[n, h], keys, vals, scale)
    return out, lse


def softmax_keyset(q_row, keys, vals, scale: float):
    """One fp64 softmax of a bf16 query row over bf16 key/value rows [n, d]."""
    lib = _load()
    q_row = np.ascontiguousarray(q_row, dtype=np.uint16)
    keys = np.ascontiguousarray(keys, dtype=np.uint16).reshape(-1, q_row.shape[-1])
    vals = np.ascontiguousarray(vals, dtype=np.uint16).reshape(-1, q_row.shape[-1])
    d = q_row.shape[-1]
    out = np.empty(d, dtype=np.float64)
    lse = np.empty(1, dtype=np.float64)
    lib.oracle_softmax_keyset(_ptr(q_row), _ptr(keys), _ptr(vals), keys.shape[0], d, d,
                              float(scale), _ptr(out), _ptr(lse))
    return out, float(lse[0])


def check_trees(parent, B: int, T: int) -> bool:
    par = np.ascontiguousarray(parent, dtype=np.int32)
    return _load().oracle_check_trees(_ptr(par), B, T) == 0


__all__ = ["verify_attn_oracle", "verify_attn_oracle_inputs", "verify_attn_oracle_packed",
           "verify_attn_oracle_window", "softmax_keyset", "check_trees",
           "max_threads", "OracleError"]
