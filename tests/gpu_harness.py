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


def out_tolerance(ref):
    """Per-element bound on |out - ref|: OUT_ATOL (1e-2) wherever bf16 can meet it.

    `out` is bf16, so rounding the exact result costs up to half a bf16 ulp: 2^-8 at
    |ref| in [1, 2), 2^-7 = 0.0078 in [2, 4), both below 1e-2; from |ref| = 4 on half an
    ulp is 2^-6 = 0.0156 and 1e-2 cannot be met. There the bound is half an ulp at |ref|
    plus the kernel's own error before that rounding. The probabilities P enter the
    tensor-core PV product as bf16 (relative error 2^-9 each); the kernel normalises by
    the sum of those rounded weights, so its output is a convex combination of the values
    whose weights are each off by at most 2 * 2^-9 relative, an error of at most
    2^-8 * |ref| when the weighted values have the sign of the result (the case for every
    |ref| >= 4 that a softmax average of the values can reach)."""
    ref = np.asarray(ref, dtype=np.float64)
    wide = 0.5 * bf16_ulp(ref) + np.abs(ref) * 2.0 ** -8
    return np.where(np.abs(ref) >= WIDEN_AT, np.maximum(OUT_ATOL, wide), OUT_ATOL)


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
