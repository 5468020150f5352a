"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that the
independent pins catch every one: the hand-worked golden example, the pure-Python
brute force, and causal attention from torch SDPA for a chain tree."""
from __future__ import annotations

import ctypes
import json
import math
import os
import subprocess

import numpy as np
import pytest

from tests.brute_force import brute_verify_attn
from tests.test_oracle import GOLDEN, _dense_reference, _small
from tree_verification_attention_longspec_b200.inputs import bf16_bits_from_f32

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "verify_attn_oracle.c")

MUTANTS = {
    "tree_mask_drops_self": ("for (int c = i; c >= 0; c = p[c]) vis[c] = 1;",
                             "for (int c = p[i]; c >= 0; c = p[c]) vis[c] = 1;"),
    "tree_mask_parent_only": ("for (int c = i; c >= 0; c = p[c]) vis[c] = 1;",
                              "vis[i] = 1; if (p[i] >= 0) vis[p[i]] = 1;"),
    "scale_missing": ("s[nk++] = scale * acc;\n      }\n      for (int t = 0;",
                      "s[nk++] = acc;\n      }\n      for (int t = 0;"),
    "lse_log2": ("const double l = m + log(sum);\n      lse[n] = l;",
                 "const double l = m + log(sum);\n      lse[n] = m + log2(sum);"),
    "gqa_modulo": ("const int kh = h / group;", "const int kh = h % Hkv;"),
    "prefix_off_by_one": ("for (int64_t j = 0; j < L; ++j) {\n        const uint16_t* kr",
                          "for (int64_t j = 1; j < L; ++j) {\n        const uint16_t* kr"),
    "tree_keys_from_batch0": ("const uint16_t* kr = k_tree + (((int64_t)b * T + t)",
                              "const uint16_t* kr = k_tree + (((int64_t)0 * T + t)"),
    "values_not_normalised": ("const double w = exp(s[nk++] - l);\n        const uint16_t* vr = v_cache",
                              "const double w = exp(s[nk++] - m);\n        const uint16_t* vr = v_cache"),
}


def _build_mutant(tmp_path, name):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    path_c = tmp_path / f"{name}.c"
    path_c.write_text(src.replace(old, new))
    path_so = tmp_path / f"{name}.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", str(path_c), "-o",
                    str(path_so), "-lm"], check=True)
    lib = ctypes.CDLL(str(path_so))
    P = ctypes.c_void_p
    lib.oracle_verify_attn.argtypes = [P] * 7 + [ctypes.c_int] * 5 + [ctypes.c_double, P,
                                                                      ctypes.c_int64, P, P, ctypes.c_int]
    lib.oracle_verify_attn.restype = ctypes.c_int
    return lib


def _run(lib, q, kc, vc, kt, vt, parent, cu, Hq, Hkv, d, T, scale):
    arrs = [np.ascontiguousarray(a, np.uint16) for a in (q, kc, vc, kt, vt)]
    par = np.ascontiguousarray(parent, np.int32)
    cu = np.ascontiguousarray(cu, np.int32)
    B = len(cu) - 1
    n = B * T * Hq
    out = np.empty((n, d))
    lse = np.empty(n)
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    rc = lib.oracle_verify_attn(*[ptr(a) for a in arrs], ptr(par), ptr(cu), B, Hq, Hkv, d, T,
                                scale, None, n, ptr(out), ptr(lse), 1)
    assert rc == 0
    return out, lse


def _pins_pass(lib) -> bool:
    """True iff the library passes all three independent pins."""
    # golden
    with open(os.path.join(GOLDEN, "hand_worked_star_tree.json")) as f:
        g = json.load(f)
    dm = g["dims"]
    bits = {k: bf16_bits_from_f32(np.asarray(g[k], dtype=np.float32))
            for k in ("q", "k_cache", "v_cache", "k_tree", "v_tree")}
    out, lse = _run(lib, bits["q"], bits["k_cache"], bits["v_cache"], bits["k_tree"], bits["v_tree"],
                    g["parent"], g["cu_seqlens"], dm["num_q_heads"], dm["num_kv_heads"],
                    dm["head_dim"], dm["tree_size"], dm["scale"])
    env = {"e": math.e, "ln": math.log, "__builtins__": {}}
    ok = np.allclose(lse, [eval(s, env) for s in g["expected_lse"]], atol=1e-12, rtol=0)
    ok &= np.allclose(out, [[eval(s, env) for s in r] for r in g["expected_out"]], atol=1e-12, rtol=0)
    # brute force, two sequences, GQA
    inp = _small(B=2, Hq=4, Hkv=2, d=8, T=10, L=None, lengths=[15, 6], tree="uniform", seed=21)
    w = inp.workload
    out, lse = _run(lib, inp.q, inp.k_cache, inp.v_cache, inp.k_tree, inp.v_tree, inp.parent,
                    inp.cu_seqlens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.tree_size, inp.scale)
    bo, bl = brute_verify_attn(inp.q, inp.k_cache, inp.v_cache, inp.k_tree, inp.v_tree, inp.parent,
                               inp.cu_seqlens, w.num_q_heads, w.num_kv_heads, w.head_dim,
                               w.tree_size, inp.scale)
    ok &= np.allclose(out, bo, atol=1e-12, rtol=0) and np.allclose(lse, bl, atol=1e-12, rtol=0)
    # chain tree vs SDPA causal
    inp = _small(B=1, Hq=4, Hkv=2, d=16, T=9, L=30, tree="chain", seed=22)
    w = inp.workload
    out, lse = _run(lib, inp.q, inp.k_cache, inp.v_cache, inp.k_tree, inp.v_tree, inp.parent,
                    inp.cu_seqlens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.tree_size, inp.scale)
    ro, rl = _dense_reference(inp, lambda b, i: np.arange(9) <= i)
    ok &= np.allclose(out, ro, atol=1e-12, rtol=0) and np.allclose(lse, rl, atol=1e-12, rtol=0)
    return bool(ok)


def test_unmodified_copy_passes(tmp_path):
    src = open(SRC).read()
    (tmp_path / "same.c").write_text(src)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                    str(tmp_path / "same.c"), "-o", str(tmp_path / "same.so"), "-lm"], check=True)
    lib = ctypes.CDLL(str(tmp_path / "same.so"))
    P = ctypes.c_void_p
    lib.oracle_verify_attn.argtypes = [P] * 7 + [ctypes.c_int] * 5 + [ctypes.c_double, P,
                                                                      ctypes.c_int64, P, P, ctypes.c_int]
    assert _pins_pass(lib)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    assert not _pins_pass(_build_mutant(tmp_path, name)), f"pins missed mutant {name}"
