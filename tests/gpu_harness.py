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


def out_tolerance(ref):
    """Per-element bound on |out - ref|: 1e-2, except where bf16 itself cannot resolve
    it. For |ref| >= 2 one bf16 ulp exceeds 2^-7 = 0.0078 and round-to-nearest alone
    costs half an ulp, so the bound there is one ulp at |ref|."""
    return np.maximum(OUT_ATOL, bf16_ulp(ref))


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


def sample_rows(inp, n_random=48, seed=0):
    """Rows r = (b*T+i)*H_q + h covering the first/last node and head of every sequence,
    the first and last row of every unit (floor(256/g) whole nodes) of every kv head,
    both ends of every 128-row query tile inside a unit, plus random rows."""
    w = inp.workload
    B, T, Hq, Hkv = w.batch, w.tree_size, w.num_q_heads, w.num_kv_heads
    g = Hq // Hkv
    tpu = 256 // g
    rows = set()
    for b in range(B):
        for i in (0, T - 1):
            for h in (0, Hq - 1):
                rows.add((b * T + i) * Hq + h)
        for kh in range(Hkv):
            for n0 in range(0, T, tpu):
                n_rows = min(tpu, T - n0) * g
                for rr in (0, 127, 128, n_rows - 1):
                    if rr < n_rows:
                        i, j = divmod(rr, g)
                        rows.add((b * T + n0 + i) * Hq + kh * g + j)
    rng = np.random.default_rng(seed)
    rows.update(int(x) for x in rng.integers(0, B * T * Hq, size=n_random))
    return np.array(sorted(rows), dtype=np.int64)
