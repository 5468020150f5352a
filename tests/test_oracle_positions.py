"""Pins of the oracle's tree positions, RoPE and bf16 rounding (oracle/tree_positions.py)
against facts fixed independently of its code: complex multiplication (RoFormer writes the
rotation of a pair as multiplication by e^{i m theta}), closed forms, invariants, brute
force and textbook tree shapes. Also: the packed per-sequence oracle against the
one-sequence oracle it is made of, and a rotated chain tree against causal attention."""
from __future__ import annotations

import math

import numpy as np
import pytest

import oracle
from oracle import tree_positions as tp
from tree_verification_attention_longspec_b200.inputs import (Workload, bfs_tree, chain_tree, make_inputs,
                                                              star_tree, window_tree)


# ----------------------------------------------------------------------------- depths
def test_depth_chain_and_star():
    assert list(tp.tree_depth_walk(chain_tree(9))) == list(range(9))
    assert list(tp.tree_depth_walk(star_tree(6))) == [0, 1, 1, 1, 1, 1]


def test_depth_equals_ancestor_count_by_closure():
    # depth(i) = number of strict ancestors, counted from the transitive closure of the
    # child->parent relation (no parent walking)
    rng = np.random.default_rng(3)
    for T in (1, 2, 7, 20, 40):
        par = bfs_tree(rng, T) if T > 3 else window_tree(rng, T, None)
        A = np.zeros((T, T), dtype=bool)
        for i in range(1, T):
            A[i, par[i]] = True
        R = A.copy()
        for k in range(T):
            R |= R[:, [k]] & R[[k], :]
        assert np.array_equal(tp.tree_depth_walk(par), R.sum(axis=1))


def test_depth_rejects_bad_trees():
    with pytest.raises(tp.BadTree):
        tp.tree_depth_walk(np.array([0, 0]))
    with pytest.raises(tp.BadTree):
        tp.tree_depth_walk(np.array([-1, 2, 1]))


def test_positions_follow_prefix_length():
    parent = np.concatenate([chain_tree(3), star_tree(4), np.zeros(0, np.int32), chain_tree(1)])
    off = np.array([0, 3, 7, 7, 8])
    cu = np.array([0, 10, 10, 15, 115])
    assert list(tp.tree_positions(parent, cu, off)) == [10, 11, 12, 0, 1, 1, 1, 100]


# ----------------------------------------------------------------------------- RoPE
def test_rope_is_complex_multiplication():
    # pair e as the complex number x[e] + i x[e + d/2], turned by e^{i pos theta^(-2e/d)}
    rng = np.random.default_rng(5)
    n, H, d, theta = 6, 3, 16, 10000.0
    x = rng.standard_normal((n, H, d))
    pos = rng.integers(0, 200000, size=n)
    z = x[..., : d // 2] + 1j * x[..., d // 2:]
    w = np.exp(1j * (pos[:, None, None] * theta ** (-2.0 * np.arange(d // 2) / d)))
    zr = z * w
    want = np.concatenate([zr.real, zr.imag], axis=-1)
    assert np.allclose(tp.rope_rotate(x, pos, theta), want, rtol=0, atol=1e-9)


def test_rope_closed_form_small():
    # d = 4, base 100: theta_0 = 1, theta_1 = 1/10; unit vectors at position 3
    x = np.zeros((1, 1, 4))
    x[0, 0, 0] = 1.0
    r = tp.rope_rotate(x, np.array([3]), 100.0)[0, 0]
    assert np.allclose(r, [math.cos(3), 0, math.sin(3), 0], atol=1e-15)
    x = np.zeros((1, 1, 4))
    x[0, 0, 3] = 1.0
    r = tp.rope_rotate(x, np.array([3]), 100.0)[0, 0]
    assert np.allclose(r, [0, -math.sin(0.3), 0, math.cos(0.3)], atol=1e-15)


def test_rope_identity_norm_and_relative_position():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((1, 1, 128))
    k = rng.standard_normal((1, 1, 128))
    assert np.array_equal(tp.rope_rotate(q, np.array([0]), 1e6), q)
    r = tp.rope_rotate(q, np.array([70001]), 1e6)
    assert abs(np.linalg.norm(r) - np.linalg.norm(q)) < 1e-12
    # <R(m) q, R(n) k> depends on m - n only
    def dot(m, n):
        return float(np.sum(tp.rope_rotate(q, np.array([m]), 5e5) * tp.rope_rotate(k, np.array([n]), 5e5)))
    a = dot(65536 + 5, 65536 + 2)
    assert abs(a - dot(5, 2)) < 1e-9 * (1 + abs(a))
    assert abs(a - dot(3, 0)) < 1e-9 * (1 + abs(a))


# ----------------------------------------------------------------------------- bf16
def test_round_to_bf16_ties_and_brute_force():
    f = tp.round_to_bf16
    # spacing of bf16 in [1, 2) is 2^-7: 1 + 2^-8 is a tie (to even: 1), 1 + 3*2^-8 too
    assert f(1 + 2.0 ** -8) == 1.0
    assert f(1 + 3 * 2.0 ** -8) == 1 + 2.0 ** -6
    assert f(-(1 + 3 * 2.0 ** -8)) == -(1 + 2.0 ** -6)
    assert f(1 + 2.0 ** -8 + 2.0 ** -30) == 1 + 2.0 ** -7
    # brute force: the nearest of the two bf16 neighbours (bit patterns around x)
    rng = np.random.default_rng(7)
    x = rng.standard_normal(4000) * 10.0 ** rng.integers(-3, 4, size=4000)
    got = f(x)
    bits = (x.astype(np.float32).view(np.uint32) >> 16).astype(np.uint64)
    for xi, gi, bi in zip(x, got, bits):
        cands = [tp.bits_to_f64(np.array([c], dtype=np.uint16))[0] for c in (bi - 1, bi, bi + 1, bi + 2)]
        dist = [abs(c - xi) for c in cands]
        best = min(dist)
        assert abs(gi - xi) == best
    assert np.array_equal(tp.bits_to_f64(tp.bf16_bits(got)), got)


# ----------------------------------------------------------------------------- oracle pieces
def test_packed_oracle_matches_one_sequence_calls_and_uniform_layout():
    # uniform trees through the packed wrapper = the batch oracle
    w = Workload("u", 3, 4, 2, 64, 5, (0, 40), "uniform")
    inp = make_inputs(w, seed=2)
    o1, l1 = oracle.verify_attn_oracle_inputs(inp)
    o2, l2 = oracle.verify_attn_oracle_packed(inp.q, inp.k_cache, inp.v_cache, inp.k_tree, inp.v_tree,
                                              inp.parent, inp.cu_seqlens, inp.node_offsets(), num_q_heads=4,
                                              num_kv_heads=2, head_dim=64, scale=inp.scale)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_rotated_chain_is_causal_attention():
    # A chain tree rotated at positions L..L+T-1 equals causal attention of the rotated
    # sequence: keys at positions 0..L-1 (given) and the new tokens, each query seeing
    # itself and everything before it. Written as a plain softmax here.
    L, T, H, d, theta = 40, 6, 2, 64, 10000.0
    rng = np.random.default_rng(9)
    def bf(shape):
        return tp.bf16_bits(tp.round_to_bf16(rng.standard_normal(shape)))
    q, kt, vt = bf((T, H, d)), bf((T, 1, d)), bf((T, 1, d))
    kc, vc = bf((L, 1, d)), bf((L, 1, d))
    parent = chain_tree(T)
    pos = tp.tree_positions(parent, np.array([0, L]), np.array([0, T]))
    assert list(pos) == list(range(L, L + T))
    qr, kr = tp.rope_bf16(q, pos, theta), tp.rope_bf16(kt, pos, theta)
    out, lse = oracle.verify_attn_oracle(qr, kc, vc, kr, vt, parent, np.array([0, L], np.int32),
                                         num_q_heads=H, num_kv_heads=1, head_dim=d, tree_size=T)
    K = np.concatenate([tp.bits_to_f64(kc)[:, 0], tp.bits_to_f64(kr)[:, 0]])
    V = np.concatenate([tp.bits_to_f64(vc)[:, 0], tp.bits_to_f64(vt)[:, 0]])
    Q = tp.bits_to_f64(qr)
    for i in range(T):
        for h in range(H):
            s = K[: L + i + 1] @ Q[i, h] / math.sqrt(d)
            m = s.max()
            ls = m + math.log(math.fsum(np.exp(s - m)))
            o = np.exp(s - ls) @ V[: L + i + 1]
            assert abs(lse[i * H + h] - ls) < 1e-12
            assert np.abs(out[i * H + h] - o).max() < 1e-12
