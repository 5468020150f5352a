"""Shared helpers for the GPU tests: move a seeded input bundle to the device, run the
C-ABI path, and pick sample rows for the oracle."""
from __future__ import annotations

import numpy as np

OUT_ATOL = 1e-2   # max-abs error on bf16 `out` against the fp64 oracle
LSE_ATOL = 1e-3   # max-abs error on fp32 `lse`


def bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (8 significant bits): 2^(floor(log2|x|) - 7)."""
    ax = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), np.finfo(np.float64).tiny)
    return np.exp2(np.floor(np.log2(ax)) - 7)


WIDEN_AT = 4.0    # |ref| from which half a bf16 ulp (2^-6 = 0.0156) exceeds OUT_ATOL


# Kernel error before the output's rounding, per unit of the values' spread: the
# probabilities P enter the tensor-core PV product rounded to bf16 (8 significant bits,
# relative error at most u = 2^-8 each) and the kernel normalises by the sum of those
# rounded weights, so its output is the convex combination sum_k w'_k v_k with
# w'_k = w_k (1 + d_k) / (1 + dbar), |d_k| <= u, dbar = sum_k w_k d_k. Its error is
# sum_k w_k (v_k - ref)(d_k - dbar) / (1 + dbar), at most 2u / (1 - u) * sum_k w_k |v_k - ref|
# (the values' mean absolute deviation under the exact weights, at most their weighted
# standard deviation, and at most sum_k w_k |v_k|, which is |ref| when the weighted
# values share the result's sign). fp32 accumulation and the exponentials (relative
# error below 1e-4) add far less.
WEIGHT_ERR = 2.0 ** -7 * 1.01


def out_tolerance(ref):
    """Per-element bound on |out - ref|: OUT_ATOL (1e-2) wherever bf16 can meet it.

    `out` is bf16, so rounding the exact result costs up to half a bf16 ulp: 2^-8 at
    |ref| in [1, 2), 2^-7 = 0.0078 in [2, 4), both below 1e-2; from |ref| = 4 on half an
    ulp is 2^-6 = 0.0156 and 1e-2 cannot be met. There the bound is half an ulp at |ref|
    plus the kernel's own error before that rounding, WEIGHT_ERR * |ref| (the case for
    every |ref| >= 4 that a softmax average of the values can reach: the weighted values
    then mostly share the result's sign)."""
    ref = np.asarray(ref, dtype=np.float64)
    wide = 0.5 * bf16_ulp(ref) + np.abs(ref) * WEIGHT_ERR
    return np.where(np.abs(ref) >= WIDEN_AT, np.maximum(OUT_ATOL, wide), OUT_ATOL)


def spread_tolerance(ref, spread):
    """The bound for inputs whose values spread widely under sharply peaked weights:
    half a bf16 ulp at |ref| plus WEIGHT_ERR times the values' weighted spread (their
    standard deviation under the exact weights, per row and dimension), never below
    out_tolerance. A fixed 1e-2 does not hold there: the weights' rounding moves the
    result by up to 2^-7 of the values' spread."""
    ref = np.asarray(ref, dtype=np.float64)
    return np.maximum(out_tolerance(ref), 0.5 * bf16_ulp(ref) + WEIGHT_ERR * np.asarray(spread) + 1e-4)


def value_spread(inp):
    """(mean, spread): per output row and dimension, the mean and the standard deviation
    of the values under the exact softmax weights of the row (fp64; prefix keys of its
    sequence and its node's ancestors-or-self in the tree), in the oracle's row order
    (b*T + i)*H_q + h. The mean is the attention output itself, which a test compares
    with the oracle's to check this helper. Test infrastructure for spread_tolerance,
    for uniform trees."""
    from tree_verification_attention_longspec_b200.inputs import bf16_bits_to_f64
    w = inp.workload
    B, T, Hq, Hkv, d = w.batch, w.tree_size, w.num_q_heads, w.num_kv_heads, w.head_dim
    g = Hq // Hkv
    q = bf16_bits_to_f64(inp.q).reshape(B, T, Hq, d)
    kc, vc = bf16_bits_to_f64(inp.k_cache), bf16_bits_to_f64(inp.v_cache)
    kt = bf16_bits_to_f64(inp.k_tree).reshape(B, T, Hkv, d)
    vt = bf16_bits_to_f64(inp.v_tree).reshape(B, T, Hkv, d)
    out = np.empty((B, T, Hq, d))
    avg = np.empty((B, T, Hq, d))
    for b in range(B):
        par = inp.parent[b * T:(b + 1) * T]
        vis = np.zeros((T, T), dtype=bool)  # vis[i, j]: node j is node i or its ancestor
        for i in range(T):
            x = i
            while x >= 0:
                vis[i, x] = True
                x = int(par[x])
        s0, s1 = int(inp.cu_seqlens[b]), int(inp.cu_seqlens[b + 1])
        for kh in range(Hkv):
            K = np.concatenate([kc[s0:s1, kh], kt[b, :, kh]])       # [L + T, d]
            V = np.concatenate([vc[s0:s1, kh], vt[b, :, kh]])
            Q = q[b, :, kh * g:(kh + 1) * g].reshape(T * g, d)      # rows (i, j)
            S = Q @ K.T * inp.scale
            mask = np.ones((T, (s1 - s0) + T), dtype=bool)
            mask[:, s1 - s0:] = vis
            S = np.where(np.repeat(mask, g, axis=0), S, -np.inf)
            W = np.exp(S - S.max(axis=1, keepdims=True))
            W /= W.sum(axis=1, keepdims=True)
            mean = W @ V
            var = np.maximum(W @ (V * V) - mean * mean, 0.0)
            out[b, :, kh * g:(kh + 1) * g] = np.sqrt(var).reshape(T, g, d)
            avg[b, :, kh * g:(kh + 1) * g] = mean.reshape(T, g, d)
    return avg.reshape(B * T * Hq, d), out.reshape(B * T * Hq, d)


def to_device(inp, device="cuda:0"):
    import torch

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)

    def i32(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)

    return dict(q=bf(inp.q), k_cache=bf(inp.k_cache), v_cache=bf(inp.v_cache), k_tree=bf(inp.k_tree),
                v_tree=bf(inp.v_tree), parent=i32(inp.parent), cu_seqlens=i32(inp.cu_seqlens))


def make_op(inp, host_lengths=True, scale=0.0, max_prefix_len=None):
    from tree_verification_attention_longspec_b200.binding import VerifyAttn
    w = inp.workload
    L = np.diff(inp.cu_seqlens)
    mpl = int(L.max()) if max_prefix_len is None else max_prefix_len
    return VerifyAttn(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.tree_size,
                      cu_seqlens_host=inp.cu_seqlens if host_lengths else None, max_prefix_len=mpl,
                      softmax_scale=scale)


def run_gpu(inp, host_lengths=True, scale=0.0, dev=None, op=None):
    """Returns (out fp64 [B*T*H_q, d], lse fp64 [B*T*H_q], device status)."""
    import torch
    if dev is None:
        dev = to_device(inp)
    if op is None:
        op = make_op(inp, host_lengths, scale)
    out, lse = op(dev["q"], dev["k_cache"], dev["v_cache"], dev["k_tree"], dev["v_tree"],
                  dev["parent"], dev["cu_seqlens"])
    torch.cuda.synchronize()
    status = op.check()
    w = inp.workload
    o = out.float().cpu().numpy().astype(np.float64).reshape(-1, w.head_dim)
    l = lse.cpu().numpy().astype(np.float64).reshape(-1)
    return o, l, status
