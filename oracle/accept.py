"""Greedy acceptance of a verified draft tree — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this module; the CUDA path never does and shares no code with it.

What it computes (LongSpec, gist.science summary: section 2C verifies the speculated
tree in one pass of the target model, which is lossless; section 3 reports the mean
acceptance length tau): with greedy decoding the target would emit, after node x, the
argmax of node x's logits. So, starting at the root (node 0, already accepted), the
draft token of a child c of the current node is accepted when it equals that argmax;
the walk moves to the smallest such child and stops when no child matches. The argmax
at the last node is the next token. The argmax is the first index of the largest value
above -inf, NaN entries skipped, 0 if a row has no such value.

Written as the plain top-down walk, one sequence at a time.
"""
from __future__ import annotations

import numpy as np


def row_argmax(row) -> int:
    """First index of the largest entry above -inf (NaN skipped); 0 if there is none."""
    best, best_i = -np.inf, 0
    for i, x in enumerate(np.asarray(row, dtype=np.float64).tolist()):
        if x > best:
            best, best_i = x, i
    return best_i


def logits_as_f64(logits, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        b = np.ascontiguousarray(logits, dtype=np.uint16)
        return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return np.asarray(logits, dtype=np.float64)


def accept_one(logits_f64, tokens, parent):
    """One tree of n nodes: returns (accepted draft count, path root first, next token),
    or (-1, [], -1) for an empty or malformed tree."""
    n = len(parent)
    if n == 0 or parent[0] != -1 or any(not (0 <= parent[i] < i) for i in range(1, n)):
        return -1, [], -1
    cur, path = 0, [0]
    while True:
        want = row_argmax(logits_f64[cur])
        nxt = None
        for c in range(cur + 1, n):  # children have larger indices; the smallest match wins
            if parent[c] == cur and tokens[c] == want:
                nxt = c
                break
        if nxt is None:
            return len(path) - 1, path, want
        cur = nxt
        path.append(cur)


def accept_greedy(inp):
    """All sequences of an ``inputs.AcceptInputs``: lists of (len, path, next)."""
    lf = logits_as_f64(inp.logits, inp.dtype)
    off = (inp.cu_tree if inp.cu_tree is not None
           else np.arange(inp.batch + 1) * inp.tree_size)
    res = []
    for b in range(inp.batch):
        s, e = int(off[b]), int(off[b + 1])
        res.append(accept_one(lf[s:e], inp.tokens[s:e], inp.parent[s:e]))
    return res


__all__ = ["row_argmax", "logits_as_f64", "accept_one", "accept_greedy"]
