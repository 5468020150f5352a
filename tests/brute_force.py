"""Pure-Python brute force for tiny cases, written independently of the C oracle.

Visibility comes from the transitive closure of the parent relation
(Floyd-Warshall on the T x T "is parent of" adjacency) instead of walking parent
links, and every sum is an exactly rounded ``math.fsum``. Only for T <= 16 and a few
dozen prefix keys.
"""
from __future__ import annotations

import math
import struct


def bf16_to_float(bits: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0]


def ancestor_closure(parent):
    """reach[i][j] is True iff tree node j is node i or an ancestor of node i."""
    T = len(parent)
    reach = [[i == j for j in range(T)] for i in range(T)]
    for i in range(T):
        p = int(parent[i])
        if p >= 0:
            reach[i][p] = True
    for k in range(T):
        for i in range(T):
            if reach[i][k]:
                rk = reach[k]
                ri = reach[i]
                for j in range(T):
                    if rk[j]:
                        ri[j] = True
    return reach


def brute_verify_attn(q, k_cache, v_cache, k_tree, v_tree, parent, cu_seqlens,
                      Hq, Hkv, d, T, scale):
    """Returns (out, lse) as nested Python lists indexed [row][c], row = (b*T+i)*Hq + h.

    Inputs are numpy uint16 bf16 bit arrays in the C-ABI layouts."""
    B = len(cu_seqlens) - 1
    g = Hq // Hkv
    out_rows, lse_rows = [], []
    qf = q.reshape(B * T, Hq, d)
    kc = k_cache.reshape(-1, Hkv, d)
    vc = v_cache.reshape(-1, Hkv, d)
    kt = k_tree.reshape(B * T, Hkv, d)
    vt = v_tree.reshape(B * T, Hkv, d)
    for b in range(B):
        reach = ancestor_closure([int(x) for x in parent[b * T:(b + 1) * T]])
        lo, hi = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
        for i in range(T):
            for h in range(Hq):
                kh = h // g
                qv = [bf16_to_float(x) for x in qf[b * T + i, h]]
                keys, vals = [], []
                for j in range(lo, hi):
                    keys.append([bf16_to_float(x) for x in kc[j, kh]])
                    vals.append([bf16_to_float(x) for x in vc[j, kh]])
                for t in range(T):
                    if reach[i][t]:
                        keys.append([bf16_to_float(x) for x in kt[b * T + t, kh]])
                        vals.append([bf16_to_float(x) for x in vt[b * T + t, kh]])
                s = [scale * math.fsum(a * c for a, c in zip(qv, kk)) for kk in keys]
                m = max(s)
                lse = m + math.log(math.fsum(math.exp(x - m) for x in s))
                w = [math.exp(x - lse) for x in s]
                o = [math.fsum(w[n] * vals[n][c] for n in range(len(vals))) for c in range(d)]
                out_rows.append(o)
                lse_rows.append(lse)
    return out_rows, lse_rows
