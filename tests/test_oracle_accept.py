"""Pins of the greedy-acceptance oracle (oracle/accept.py): a hand-worked example
(tests/golden/hand_worked_accept.json), the argmax rule against numpy's first-occurrence
argmax, and a bottom-up brute force (every node whose whole root path matches, the deepest
one wins) on random trees whose siblings carry distinct tokens."""
from __future__ import annotations

import json
import os

import numpy as np

from oracle import accept as oa
from tree_verification_attention_longspec_b200.inputs import (AcceptInputs, bf16_bits_from_f32, draw_tree,
                                                              make_accept_inputs)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_accept.json")


def _golden_inputs():
    with open(GOLDEN) as f:
        g = json.load(f)
    logits = np.array([[float(x) for x in row] for row in g["logits"]], dtype=np.float32)
    inp = AcceptInputs(logits, np.array(g["tokens"], np.int32), np.array(g["parent"], np.int32),
                       np.array(g["cu_tree"], np.int32), len(g["cu_tree"]) - 1, g["tree_size"], g["vocab"], "f32")
    return g, inp


def test_hand_worked_example():
    g, inp = _golden_inputs()
    got = oa.accept_greedy(inp)
    for (n, path, nxt), want in zip(got, g["expected"]):
        assert n == want["accept_len"] and path == want["path"] and nxt == want["next_token"]
    # the same values as bf16 (all exactly representable)
    inp.logits = bf16_bits_from_f32(inp.logits)
    inp.dtype = "bf16"
    assert oa.accept_greedy(inp) == got


def test_row_argmax_matches_numpy_first_occurrence():
    rng = np.random.default_rng(0)
    for _ in range(200):
        row = rng.integers(-3, 4, size=rng.integers(1, 40)).astype(np.float64)  # many ties
        assert oa.row_argmax(row) == int(np.argmax(row))
        r2 = row.copy()
        r2[rng.random(len(r2)) < 0.3] = np.nan
        if np.isnan(r2).all():
            assert oa.row_argmax(r2) == 0
        else:
            assert oa.row_argmax(r2) == int(np.nanargmax(r2))
    assert oa.row_argmax([-np.inf, -np.inf]) == 0
    assert oa.row_argmax([-np.inf, -5.0, -np.inf]) == 1


def _distinct_sibling_tokens(rng, parent, vocab, peak, p):
    tok = rng.integers(0, vocab, size=len(parent)).astype(np.int32)
    for i in range(1, len(parent)):
        if rng.random() < p:
            tok[i] = peak[parent[i]]
    # make siblings distinct: a repeated token moves to a fresh value
    for x in range(len(parent)):
        seen = set()
        for c in range(x + 1, len(parent)):
            if parent[c] == x:
                while int(tok[c]) in seen:
                    tok[c] = (tok[c] + 1) % vocab
                seen.add(int(tok[c]))
    return tok


def test_brute_force_deepest_fully_matching_node():
    rng = np.random.default_rng(1)
    for trial in range(60):
        T = int(rng.integers(1, 40))
        vocab = int(rng.integers(T + 2, 3 * T + 10))
        parent = draw_tree(["uniform", "window8", "bfs", "chain", "star"][trial % 5], rng, T)
        logits = rng.standard_normal((T, vocab))
        peak = np.argmax(logits, axis=1)
        tok = _distinct_sibling_tokens(rng, parent, vocab, peak, 0.8)
        n, path, nxt = oa.accept_one(logits, tok, parent)
        # bottom-up: node i is reachable when every node on its path (root excluded)
        # carries its parent's argmax
        ok = []
        for i in range(T):
            x, good = i, True
            while x != 0:
                if tok[x] != np.argmax(logits[parent[x]]):
                    good = False
                    break
                x = parent[x]
            ok.append(good)
        depth = [0] * T
        for i in range(1, T):
            depth[i] = depth[parent[i]] + 1
        deepest = max((i for i in range(T) if ok[i]), key=lambda i: depth[i])
        chain = []
        x = deepest
        while x != -1:
            chain.append(x)
            x = parent[x] if x != 0 else -1
        assert path == chain[::-1] and n == depth[deepest] and nxt == int(np.argmax(logits[deepest]))


def test_generator_plants_walks():
    inp = make_accept_inputs(2, 32, 1000, "f32", match_prob=0.9, seed=3)
    lens = [r[0] for r in oa.accept_greedy(inp)]
    assert max(lens) >= 2  # the planted peaks make multi-step walks likely
