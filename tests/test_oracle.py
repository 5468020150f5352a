"""Pins for the fp64 oracle, each against something other than the oracle itself.

What the LongSpec pages fix (gist.science summary, section 2C; abstracts): the
prefix is attended with no mask, the tree under a tree mask, and the log-sum-exp
join is exact, so the verification result is one softmax over the union. The
pins below are chosen so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one of them.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tests.brute_force import ancestor_closure, brute_verify_attn
from tree_verification_attention_longspec_b200.inputs import (
    Workload, bf16_bits_from_f32, bf16_bits_to_f64, bfs_tree, chain_tree, make_inputs, star_tree,
    tree_depths, window_tree)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _small(B=1, Hq=4, Hkv=2, d=16, T=8, L=24, tree="uniform", seed=0, lengths=None, scale=1.0):
    w = Workload("t", B, Hq, Hkv, d, T, L, tree, input_scale=scale, lengths=lengths)
    return make_inputs(w, seed=seed)


def _oracle(inp, **kw):
    return oracle.verify_attn_oracle_inputs(inp, **kw)


def _dense_reference(inp, vis_fn):
    """Independent dense attention with an explicit boolean mask, using torch's
    scaled_dot_product_attention in float64 (library routine) for `out` and a masked
    logsumexp for `lse`. vis_fn(b, i) -> bool array over the T tree nodes."""
    w = inp.workload
    B, T, Hq, Hkv, d = w.batch, w.tree_size, w.num_q_heads, w.num_kv_heads, w.head_dim
    g = Hq // Hkv
    q = torch.from_numpy(bf16_bits_to_f64(inp.q)).reshape(B, T, Hq, d)
    kc = torch.from_numpy(bf16_bits_to_f64(inp.k_cache)).reshape(-1, Hkv, d)
    vc = torch.from_numpy(bf16_bits_to_f64(inp.v_cache)).reshape(-1, Hkv, d)
    kt = torch.from_numpy(bf16_bits_to_f64(inp.k_tree)).reshape(B, T, Hkv, d)
    vt = torch.from_numpy(bf16_bits_to_f64(inp.v_tree)).reshape(B, T, Hkv, d)
    outs, lses = [], []
    for b in range(B):
        lo, hi = int(inp.cu_seqlens[b]), int(inp.cu_seqlens[b + 1])
        K = torch.cat([kc[lo:hi], kt[b]], 0)             # [L+T, Hkv, d]
        V = torch.cat([vc[lo:hi], vt[b]], 0)
        L = hi - lo
        mask = torch.zeros(T, L + T, dtype=torch.bool)
        mask[:, :L] = True
        for i in range(T):
            mask[i, L:] = torch.from_numpy(np.asarray(vis_fn(b, i), dtype=bool))
        Kh = K.permute(1, 0, 2).repeat_interleave(g, 0)   # [Hq, L+T, d]
        Vh = V.permute(1, 0, 2).repeat_interleave(g, 0)
        Q = q[b].permute(1, 0, 2)                           # [Hq, T, d]
        o = torch.nn.functional.scaled_dot_product_attention(
            Q, Kh, Vh, attn_mask=mask, scale=inp.scale)     # [Hq, T, d]
        sc = (Q @ Kh.transpose(1, 2)) * inp.scale
        lse = torch.logsumexp(sc.masked_fill(~mask, -math.inf), dim=-1)  # [Hq, T]
        outs.append(o.permute(1, 0, 2).reshape(T * Hq, d))
        lses.append(lse.permute(1, 0).reshape(T * Hq))
    return torch.cat(outs).numpy(), torch.cat(lses).numpy()


# ----------------------------------------------------------------------------- golden
def test_hand_worked_star_tree():
    with open(os.path.join(GOLDEN, "hand_worked_star_tree.json")) as f:
        g = json.load(f)
    dims = g["dims"]
    bits = {k: bf16_bits_from_f32(np.asarray(g[k], dtype=np.float32))
            for k in ("q", "k_cache", "v_cache", "k_tree", "v_tree")}
    out, lse = oracle.verify_attn_oracle(
        bits["q"], bits["k_cache"], bits["v_cache"], bits["k_tree"], bits["v_tree"],
        np.asarray(g["parent"], np.int32), np.asarray(g["cu_seqlens"], np.int32),
        num_q_heads=dims["num_q_heads"], num_kv_heads=dims["num_kv_heads"],
        head_dim=dims["head_dim"], tree_size=dims["tree_size"], scale=dims["scale"])
    env = {"e": math.e, "ln": math.log, "__builtins__": {}}
    exp_lse = np.array([eval(s, env) for s in g["expected_lse"]])
    exp_out = np.array([[eval(s, env) for s in row] for row in g["expected_out"]])
    np.testing.assert_allclose(lse, exp_lse, rtol=0, atol=1e-14)
    np.testing.assert_allclose(out, exp_out, rtol=0, atol=1e-14)


# ----------------------------------------------------------------------------- (1) chain -> causal
@pytest.mark.parametrize("B,L,T,Hq,Hkv,d", [(1, 40, 12, 4, 2, 16), (2, 17, 7, 6, 3, 8), (1, 0, 5, 2, 1, 8)])
def test_chain_tree_is_causal_attention(B, L, T, Hq, Hkv, d):
    """parent[i] = i-1 turns the tree into a sequence: the result must be causal
    attention of queries at positions L..L+T-1 over keys 0..L+T-1 (bottom-right
    aligned), computed here by torch SDPA in fp64 with an explicit causal mask."""
    inp = _small(B=B, Hq=Hq, Hkv=Hkv, d=d, T=T, L=L, tree="chain", seed=3)
    out, lse = _oracle(inp)
    ref_out, ref_lse = _dense_reference(inp, lambda b, i: np.arange(T) <= i)
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_textbook_causal_softmax_agrees():
    """Chain tree against a causal softmax written out with numpy loops (no torch)."""
    inp = _small(B=1, Hq=2, Hkv=1, d=8, T=6, L=10, tree="chain", seed=5)
    out, lse = _oracle(inp)
    q = bf16_bits_to_f64(inp.q).reshape(6, 2, 8)
    K = np.concatenate([bf16_bits_to_f64(inp.k_cache).reshape(10, 8),
                        bf16_bits_to_f64(inp.k_tree).reshape(6, 8)])
    V = np.concatenate([bf16_bits_to_f64(inp.v_cache).reshape(10, 8),
                        bf16_bits_to_f64(inp.v_tree).reshape(6, 8)])
    r = 0
    for i in range(6):
        for h in range(2):
            n = 10 + i + 1                      # keys at positions 0 .. L+i
            s = np.array([inp.scale * float(np.dot(q[i, h], K[j])) for j in range(n)])
            ex = np.exp(s - s.max())
            assert abs(lse[r] - (s.max() + math.log(ex.sum()))) < 1e-12
            np.testing.assert_allclose(out[r], (ex[:, None] * V[:n]).sum(0) / ex.sum(), atol=1e-12)
            r += 1


# ----------------------------------------------------------------------------- (2) merge identity
@pytest.mark.parametrize("splits", [1, 3, 7])
def test_lse_merge_of_partials_equals_union(splits):
    """Partial softmaxes over disjoint key sets (prefix slices and the visible tree
    nodes), merged by lse = ln sum exp(lse_x), out = sum exp(lse_x - lse) out_x, must
    equal the oracle's single union softmax (the 'Aggregation' step of section 2C)."""
    inp = _small(B=2, Hq=4, Hkv=2, d=16, T=8, L=None, lengths=[37, 5], tree="uniform", seed=11)
    out, lse = _oracle(inp)
    w = inp.workload
    B, T, Hq, Hkv, d = w.batch, w.tree_size, w.num_q_heads, w.num_kv_heads, w.head_dim
    g = Hq // Hkv
    kc = inp.k_cache.reshape(-1, Hkv, d)
    vc = inp.v_cache.reshape(-1, Hkv, d)
    kt = inp.k_tree.reshape(B * T, Hkv, d)
    vt = inp.v_tree.reshape(B * T, Hkv, d)
    qv = inp.q.reshape(B * T, Hq, d)
    for r in range(B * T * Hq):
        h, tok = r % Hq, r // Hq
        b, i = tok // T, tok % T
        kh = h // g
        lo, hi = int(inp.cu_seqlens[b]), int(inp.cu_seqlens[b + 1])
        bounds = np.linspace(lo, hi, splits + 1).astype(int)
        parts = [oracle.softmax_keyset(qv[tok, h], kc[a:c, kh], vc[a:c, kh], inp.scale)
                 for a, c in zip(bounds[:-1], bounds[1:])]
        anc = [t for t in range(T) if ancestor_closure(list(inp.parent[b * T:(b + 1) * T]))[i][t]]
        parts.append(oracle.softmax_keyset(qv[tok, h], kt[b * T + np.array(anc), kh],
                                           vt[b * T + np.array(anc), kh], inp.scale))
        lses = np.array([p[1] for p in parts])
        mx = lses.max()
        tot = mx + math.log(sum(math.exp(x - mx) for x in lses if x > -math.inf))
        merged = sum(math.exp(p[1] - tot) * p[0] for p in parts if p[1] > -math.inf)
        assert abs(tot - lse[r]) < 1e-12
        np.testing.assert_allclose(merged, out[r], rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- (3) equal keys
def test_equal_keys_give_mean_of_visible_values():
    """All keys of a kv head identical: every visible key has the same score, so out
    is the mean of the visible values and lse = scale*<q,k> + ln(L_b + depth(i) + 1)."""
    inp = _small(B=2, Hq=6, Hkv=2, d=16, T=10, L=None, lengths=[13, 29], tree="uniform", seed=7)
    w = inp.workload
    B, T, Hq, Hkv, d = w.batch, w.tree_size, w.num_q_heads, w.num_kv_heads, w.head_dim
    rng = np.random.default_rng(99)
    kvec = bf16_bits_from_f32(rng.standard_normal((Hkv, d)).astype(np.float32))
    inp.k_cache = np.broadcast_to(kvec, inp.k_cache.shape).copy()
    inp.k_tree = np.broadcast_to(kvec, inp.k_tree.shape).copy()
    out, lse = _oracle(inp)
    q = bf16_bits_to_f64(inp.q).reshape(B * T, Hq, d)
    k = bf16_bits_to_f64(kvec)
    vc = bf16_bits_to_f64(inp.v_cache).reshape(-1, Hkv, d)
    vt = bf16_bits_to_f64(inp.v_tree).reshape(B * T, Hkv, d)
    for b in range(B):
        par = inp.parent[b * T:(b + 1) * T]
        depth = tree_depths(par)
        lo, hi = int(inp.cu_seqlens[b]), int(inp.cu_seqlens[b + 1])
        for i in range(T):
            path = []
            c = i
            while c >= 0:
                path.append(c)
                c = par[c]
            assert len(path) == depth[i] + 1
            for h in range(Hq):
                kh = h // (Hq // Hkv)
                r = (b * T + i) * Hq + h
                n = (hi - lo) + depth[i] + 1
                exp_lse = inp.scale * float(np.dot(q[b * T + i, h], k[kh])) + math.log(n)
                exp_out = (vc[lo:hi, kh].sum(0) + vt[b * T + np.array(path), kh].sum(0)) / n
                assert abs(lse[r] - exp_lse) < 1e-12
                np.testing.assert_allclose(out[r], exp_out, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- (4) brute force
@pytest.mark.parametrize("tree,seed", [("uniform", 0), ("uniform", 1), ("window8", 2), ("bfs", 3),
                                       ("chain", 4), ("star", 5)])
def test_brute_force_tiny(tree, seed):
    B = 2
    inp = _small(B=B, Hq=4, Hkv=2, d=8, T=12, L=None, lengths=[20, 9], tree=tree, seed=seed)
    out, lse = _oracle(inp)
    w = inp.workload
    bo, bl = brute_verify_attn(inp.q, inp.k_cache, inp.v_cache, inp.k_tree, inp.v_tree,
                               inp.parent, inp.cu_seqlens, w.num_q_heads, w.num_kv_heads,
                               w.head_dim, w.tree_size, inp.scale)
    np.testing.assert_allclose(out, np.array(bo), rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, np.array(bl), rtol=0, atol=1e-13)


def test_brute_force_random_trees_all_shapes():
    """Every tree on 6 nodes in topological numbering is drawn by some parent vector;
    sweep 40 random ones, including T = 1."""
    rng = np.random.default_rng(123)
    for trial in range(40):
        T = int(rng.integers(1, 7))
        par = np.array([-1] + [int(rng.integers(0, i)) for i in range(1, T)], dtype=np.int32)
        w = Workload("x", 1, 2, 1, 4, T, int(rng.integers(0, 6)), "chain")
        inp = make_inputs(w, seed=trial)
        inp.parent = par
        out, lse = _oracle(inp)
        bo, bl = brute_verify_attn(inp.q, inp.k_cache, inp.v_cache, inp.k_tree, inp.v_tree,
                                   inp.parent, inp.cu_seqlens, 2, 1, 4, T, inp.scale)
        np.testing.assert_allclose(out, np.array(bo), rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse, np.array(bl), rtol=0, atol=1e-13)


# ----------------------------------------------------------------------------- (5) invariants
def test_constant_values_give_constant_output():
    inp = _small(B=1, Hq=4, Hkv=1, d=16, T=9, L=31, tree="uniform", seed=2)
    one = bf16_bits_from_f32(np.ones(1, np.float32))[0]
    inp.v_cache[:] = one
    inp.v_tree[:] = one
    out, _ = _oracle(inp)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-13)


def test_prefix_permutation_invariance():
    inp = _small(B=1, Hq=4, Hkv=2, d=16, T=8, L=50, tree="uniform", seed=4)
    out, lse = _oracle(inp)
    perm = np.random.default_rng(1).permutation(50)
    inp.k_cache = inp.k_cache[perm].copy()
    inp.v_cache = inp.v_cache[perm].copy()
    out2, lse2 = _oracle(inp)
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-12)


def test_topological_relabelling_permutes_rows():
    """Renumber the tree nodes by another topological order: rows move with the nodes."""
    T, Hq = 10, 4
    inp = _small(B=1, Hq=Hq, Hkv=2, d=8, T=T, L=15, tree="uniform", seed=8)
    out, lse = _oracle(inp)
    par = inp.parent
    # a random topological order: repeatedly pick any node whose parent is placed
    rng = np.random.default_rng(5)
    placed, order = set(), []
    while len(order) < T:
        ready = [n for n in range(T) if n not in placed and (par[n] < 0 or par[n] in placed)]
        n = int(rng.choice(ready))
        placed.add(n)
        order.append(n)
    new_of = {old: new for new, old in enumerate(order)}
    new_par = np.array([-1 if par[o] < 0 else new_of[int(par[o])] for o in order], np.int32)
    inp2 = _small(B=1, Hq=Hq, Hkv=2, d=8, T=T, L=15, tree="uniform", seed=8)
    o = np.array(order)
    inp2.parent = new_par
    inp2.q = inp.q[o].copy()
    inp2.k_tree = inp.k_tree[o].copy()
    inp2.v_tree = inp.v_tree[o].copy()
    out2, lse2 = _oracle(inp2)
    rows_new = np.array([new_of[i] * Hq + h for i in range(T) for h in range(Hq)])
    np.testing.assert_allclose(out2[rows_new], out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2[rows_new], lse, rtol=0, atol=1e-12)


def test_star_tree_sees_prefix_root_and_self():
    T = 7
    inp = _small(B=1, Hq=2, Hkv=1, d=8, T=T, L=12, tree="star", seed=9)
    out, lse = _oracle(inp)
    ref_out, ref_lse = _dense_reference(inp, lambda b, i: np.isin(np.arange(T), [0, i]))
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_single_node_tree_is_decode_attention():
    inp = _small(B=3, Hq=4, Hkv=2, d=16, T=1, L=None, lengths=[7, 0, 33], tree="chain", seed=10)
    out, lse = _oracle(inp)
    ref_out, ref_lse = _dense_reference(inp, lambda b, i: np.array([True]))
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_empty_prefix_is_pure_tree_attention():
    inp = _small(B=2, Hq=4, Hkv=2, d=8, T=9, L=0, tree="uniform", seed=12)
    out, lse = _oracle(inp)
    reach = [ancestor_closure(list(inp.parent[b * 9:(b + 1) * 9])) for b in range(2)]
    ref_out, ref_lse = _dense_reference(inp, lambda b, i: np.array(reach[b][i]))
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_key_shift_moves_lse_only():
    """Adding one vector c to every key adds scale*<q_i, c> to every score of row i:
    lse shifts by exactly that, out is unchanged. Keys and c are multiples of 1/8
    small enough that k + c is exact in bf16, so the check is exact in fp64."""
    T, L, d, Hq, Hkv = 6, 20, 8, 4, 2
    inp = _small(B=1, Hq=Hq, Hkv=Hkv, d=d, T=T, L=L, tree="uniform", seed=13)
    rng = np.random.default_rng(3)
    kc = rng.integers(-64, 65, size=(L, Hkv, d)).astype(np.float32) / 8
    kt = rng.integers(-64, 65, size=(T, Hkv, d)).astype(np.float32) / 8
    c = rng.integers(-32, 33, size=(Hkv, d)).astype(np.float32) / 8
    inp.k_cache, inp.k_tree = bf16_bits_from_f32(kc), bf16_bits_from_f32(kt)
    out, lse = _oracle(inp)
    inp.k_cache, inp.k_tree = bf16_bits_from_f32(kc + c), bf16_bits_from_f32(kt + c)
    out2, lse2 = _oracle(inp)
    q = bf16_bits_to_f64(inp.q).reshape(T, Hq, d)
    g = Hq // Hkv
    delta = np.array([inp.scale * float(np.dot(q[i, h], c[h // g].astype(np.float64)))
                      for i in range(T) for h in range(Hq)])
    np.testing.assert_allclose(lse2 - lse, delta, rtol=0, atol=1e-11)
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-11)


def test_bad_trees_rejected():
    good = chain_tree(5)
    assert oracle.check_trees(good, 1, 5)
    for bad in ([0, 0, 1, 2, 3], [-1, 1, 1, 2, 3], [-1, 0, 3, 2, 3], [-1, -1, 0, 1, 2]):
        assert not oracle.check_trees(np.array(bad, np.int32), 1, 5)
    inp = _small(T=5, tree="chain")
    inp.parent = np.array([-1, 0, 2, 1, 3], np.int32)
    with pytest.raises(oracle.OracleError):
        _oracle(inp)


def test_row_subset_matches_full():
    inp = _small(B=2, Hq=4, Hkv=2, d=16, T=8, L=None, lengths=[19, 40], tree="window8", seed=14)
    out, lse = _oracle(inp)
    rows = np.array([0, 5, 17, 63, 31, 2])
    o2, l2 = _oracle(inp, rows=rows)
    np.testing.assert_array_equal(o2, out[rows])
    np.testing.assert_array_equal(l2, lse[rows])


def test_generators_shapes():
    """Tree generators: parents precede children; bfs depth <= 12 and branching <= 4."""
    rng = np.random.default_rng(0)
    for _ in range(20):
        p = bfs_tree(rng, 128)
        assert p[0] == -1 and all(0 <= p[i] < i for i in range(1, 128))
        assert tree_depths(p).max() <= 12
        assert np.bincount(p[1:], minlength=128).max() <= 4
        w8 = window_tree(rng, 64, 8)
        assert all(max(0, i - 8) <= w8[i] < i for i in range(1, 64))
    assert list(star_tree(4)) == [-1, 0, 0, 0]
