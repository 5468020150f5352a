"""Pins of the sliding-window oracle (oracle.verify_attn_oracle_window): a window that
covers everything equals the plain (C) oracle; a chain tree under a window equals causal
sliding-window attention written as a plain softmax over the last W positions; a window of
one position leaves each node only itself."""
from __future__ import annotations

import math

import numpy as np

import oracle
from oracle import tree_positions as tp
from tree_verification_attention_longspec_b200.inputs import Workload, make_inputs


def _win(inp, window, rows=None):
    w = inp.workload
    return oracle.verify_attn_oracle_window(inp.q, inp.k_cache, inp.v_cache, inp.k_tree, inp.v_tree, inp.parent,
                                            inp.cu_seqlens, inp.node_offsets(), num_q_heads=w.num_q_heads,
                                            num_kv_heads=w.num_kv_heads, head_dim=w.head_dim, scale=inp.scale,
                                            window=window, rows=rows)


def test_wide_window_is_the_plain_oracle():
    w = Workload("wwide", 3, 4, 2, 64, 9, 0, "bfs", lengths=[50, 0, 130], tree_sizes=[9, 4, 1])
    inp = make_inputs(w, seed=1)
    o, l_ = _win(inp, 10_000)
    ro, rl = oracle.verify_attn_oracle_packed(inp.q, inp.k_cache, inp.v_cache, inp.k_tree, inp.v_tree, inp.parent,
                                              inp.cu_seqlens, inp.node_offsets(), num_q_heads=4, num_kv_heads=2,
                                              head_dim=64, scale=inp.scale)
    assert np.abs(o - ro).max() < 1e-12 and np.abs(l_ - rl).max() < 1e-12


def test_chain_under_window_is_causal_sliding_window():
    L, T, W, H, d = 40, 7, 12, 2, 64
    w = Workload("wchain", 1, H, 1, d, T, L, "chain")
    inp = make_inputs(w, seed=2)
    o, l_ = _win(inp, W)
    K = np.concatenate([tp.bits_to_f64(inp.k_cache)[:, 0], tp.bits_to_f64(inp.k_tree)[:, 0]])
    V = np.concatenate([tp.bits_to_f64(inp.v_cache)[:, 0], tp.bits_to_f64(inp.v_tree)[:, 0]])
    Q = tp.bits_to_f64(inp.q)
    for i in range(T):
        P = L + i  # position of node i; keys at positions P-W+1..P
        for h in range(H):
            s = K[P - W + 1: P + 1] @ Q[i, h] / math.sqrt(d)
            m = s.max()
            ls = m + math.log(math.fsum(np.exp(s - m)))
            ref = np.exp(s - ls) @ V[P - W + 1: P + 1]
            assert abs(l_[i * H + h] - ls) < 1e-12
            assert np.abs(o[i * H + h] - ref).max() < 1e-12


def test_window_of_one_sees_only_itself():
    w = Workload("wone", 2, 2, 1, 64, 1, 30, "chain")
    inp = make_inputs(w, seed=3)
    o, l_ = _win(inp, 1)
    V = tp.bits_to_f64(inp.v_tree)[:, 0]
    Kt = tp.bits_to_f64(inp.k_tree)[:, 0]
    Q = tp.bits_to_f64(inp.q)
    for n in range(2):
        for h in range(2):
            assert np.abs(o[n * 2 + h] - V[n]).max() < 1e-15
            assert abs(l_[n * 2 + h] - Q[n, h] @ Kt[n] / 8.0) < 1e-12
