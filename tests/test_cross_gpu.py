"""GPU parity of prefix-only attention (ls_cross_attn, the draft model's cross-attention
over the target's KV cache) against the fp64 oracle: each query row's softmax over exactly
the prefix keys of its sequence (oracle.softmax_keyset), no tree keys."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_harness import LSE_ATOL, out_tolerance, to_device
from tree_verification_attention_longspec_b200 import binding
from tree_verification_attention_longspec_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu


def _oracle_rows(inp, rows):
    w = inp.workload
    g = w.num_q_heads // w.num_kv_heads
    cu = inp.cu_seqlens
    out = np.zeros((len(rows), w.head_dim))
    lse = np.zeros(len(rows))
    for n, r in enumerate(rows):
        tok, h = divmod(int(r), w.num_q_heads)
        b = tok // w.tree_size
        kh = h // g
        keys = inp.k_cache[cu[b]:cu[b + 1], kh]
        vals = inp.v_cache[cu[b]:cu[b + 1], kh]
        out[n], lse[n] = oracle.softmax_keyset(inp.q[tok, h], keys, vals, inp.scale)
    return out, lse


def _run(inp, uniform=False):
    w = inp.workload
    dev = to_device(inp)
    L = np.diff(inp.cu_seqlens)
    dims, keep = binding.make_dims(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.tree_size,
                                   max_prefix_len=int(L.max()) if len(L) else 0,
                                   cu_seqlens_host=None if uniform else inp.cu_seqlens)
    wsb = binding.cross_workspace_size(dims)
    assert wsb > 0
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    out = torch.full_like(dev["q"], float("nan"))
    lse = torch.full((out.shape[0], w.num_q_heads), float("nan"), dtype=torch.float32, device="cuda")
    kc = dev["k_cache"].data_ptr() if dev["k_cache"].numel() else None
    vc = dev["v_cache"].data_ptr() if dev["v_cache"].numel() else None
    stream = torch.cuda.current_stream().cuda_stream
    rc = binding.call_cross_raw(dev["q"].data_ptr(), kc, vc, dev["cu_seqlens"].data_ptr(), out.data_ptr(),
                                lse.data_ptr(), dims, ws.data_ptr(), wsb, stream)
    assert rc == binding.LS_OK
    torch.cuda.synchronize()
    assert binding.check(dims, ws.data_ptr(), stream) == 0
    o = out.float().cpu().numpy().astype(np.float64).reshape(-1, w.head_dim)
    l_ = lse.cpu().numpy().astype(np.float64).reshape(-1)
    return o, l_


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [1, 4, 33])
def test_cross_small_all_rows(d, T):
    # lengths off block boundaries, one shorter than a block, an empty sequence
    w = Workload("cross", 4, 8, 2, d, T, 0, "chain", input_scale=1.0, lengths=[1000, 37, 0, 2500])
    inp = make_inputs(w, seed=11)
    o, l_ = _run(inp)
    rows = np.arange(o.shape[0])
    ro, rl = _oracle_rows(inp, rows)
    L = np.diff(inp.cu_seqlens)
    empty = np.repeat(L == 0, T * w.num_q_heads)  # rows of sequences without keys
    assert np.all(o[empty] == 0) and np.all(np.isneginf(l_[empty]))
    keep = ~empty
    assert np.all(np.isfinite(o[keep])) and np.all(np.isfinite(l_[keep]))
    assert np.all(np.abs(o[keep] - ro[keep]) <= out_tolerance(ro[keep]))
    assert np.abs(l_[keep] - rl[keep]).max() <= LSE_ATOL


def test_cross_uniform_plan():
    w = Workload("cross_uniform", 3, 12, 4, 128, 2, 0, "chain", input_scale=1.0, lengths=[3000, 128, 700])
    inp = make_inputs(w, seed=12)
    o, l_ = _run(inp, uniform=True)
    rows = np.arange(o.shape[0])
    ro, rl = _oracle_rows(inp, rows)
    assert np.all(np.abs(o - ro) <= out_tolerance(ro))
    assert np.abs(l_ - rl).max() <= LSE_ATOL


def test_cross_long_prefix_all_rows():
    # one draft query per step over a Qwen2.5-7B-shaped 64k cache
    w = Workload("cross_qwen", 1, 28, 4, 128, 1, 65536, "chain", input_scale=1.0)
    inp = make_inputs(w, seed=0)
    o, l_ = _run(inp)
    rows = np.arange(o.shape[0])
    ro, rl = _oracle_rows(inp, rows)
    assert np.all(np.abs(o[rows] - ro) <= out_tolerance(ro))
    assert np.abs(l_[rows] - rl).max() <= LSE_ATOL


def test_cross_without_any_key():
    w = Workload("cross_empty", 2, 4, 1, 64, 3, 0, "chain", input_scale=1.0, lengths=[0, 0])
    inp = make_inputs(w, seed=13)
    o, l_ = _run(inp)
    assert np.all(o == 0) and np.all(np.isneginf(l_))
