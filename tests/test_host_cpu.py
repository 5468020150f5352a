"""CPU-only checks of the host side: the chunk plan, the C-ABI library's exports and
its argument checks that return before any device work."""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "tree_verification_attention_longspec_b200", "csrc")
HEADER = os.path.join(ROOT, "include", "ls_verify_attn.h")


@pytest.fixture(scope="module")
def plan_check(tmp_path_factory):
    exe = tmp_path_factory.mktemp("plan") / "plan_check"
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", CSRC, os.path.join(ROOT, "tests", "plan_check.cpp"),
                    "-o", str(exe)], check=True)
    return str(exe)


@pytest.mark.parametrize("B,Hq,Hkv,T,C,uniform,lengths", [
    (1, 28, 4, 64, 29, -1, [65536]),
    (1, 32, 8, 64, 7, -1, [16384]),
    (1, 64, 8, 128, 56, -1, [131072]),
    (1, 4, 1, 16, 3, -1, [1024]),
    (8, 32, 8, 64, 40, -1, [4096, 32768, 5000, 1, 0, 128, 129, 20000]),
    (3, 6, 3, 5, 2, -1, [0, 0, 0]),
    (4, 8, 2, 33, 5, 4, [1200, 17, 0, 1920]),   # uniform plan: max 1920 -> 15 prefix + 1 tree block -> 4 chunks of 5
    (2, 64, 1, 128, 1, -1, [300, 1]),            # g = 64: 4 nodes per unit, 32 units per kv head
])
def test_chunk_plan_covers_every_block_once(plan_check, B, Hq, Hkv, T, C, uniform, lengths):
    r = subprocess.run([plan_check, str(B), str(Hq), str(Hkv), str(T), str(C), str(uniform),
                        *map(str, lengths)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr


@pytest.mark.parametrize("B,Hq,Hkv,T,C,uniform,lengths", [
    (1, 28, 4, 1, 14, -1, [65536]),
    (3, 8, 2, 4, 3, -1, [0, 129, 1000]),
    (2, 8, 8, 1, 5, 2, [640, 7]),
])
def test_prefix_only_plan_covers_every_prefix_block_once(plan_check, B, Hq, Hkv, T, C, uniform, lengths):
    # cross-attention plans: the key lists hold the prefix blocks only (no tree block)
    env = dict(os.environ, PLAN_CHECK_NO_TREE="1")
    r = subprocess.run([plan_check, str(B), str(Hq), str(Hkv), str(T), str(C), str(uniform),
                        *map(str, lengths)], capture_output=True, text=True, env=env)
    assert r.returncode == 0, r.stdout + r.stderr


def test_plan_check_catches_a_plan_too_short_for_the_keys(plan_check):
    # uniform plan of 3 chunks of 5 blocks: 1920 keys need 15 prefix blocks and the tree
    # block, 16 in all; spread evenly over 3 chunks one of them needs 6 blocks, more than
    # the plan's C (on the device the combine reports such lengths as LS_ERR_LENGTHS)
    r = subprocess.run([plan_check, "1", "4", "1", "16", "5", "3", "1920"], capture_output=True, text=True)
    assert r.returncode == 1 and "too long" in r.stdout


def test_plan_check_catches_a_missing_block(plan_check):
    # a prefix-only plan of one chunk of 5 blocks over 6 blocks of keys: the sixth block is
    # covered by no chunk (the even split of 6 blocks over 1 chunk is 6 > C first)
    env = dict(os.environ, PLAN_CHECK_NO_TREE="1")
    r = subprocess.run([plan_check, "1", "4", "1", "16", "5", "1", "700"], capture_output=True, text=True, env=env)
    assert r.returncode == 1 and ("too long" in r.stdout or "covered 0 times" in r.stdout)


def test_random_plans(plan_check):
    rng = np.random.default_rng(0)
    for _ in range(25):
        B = int(rng.integers(1, 6))
        Hkv = int(rng.integers(1, 5))
        Hq = Hkv * int(rng.integers(1, 9))
        T = int(rng.integers(1, 129))
        lengths = rng.integers(0, 3000, size=B)
        C = int(rng.integers(1, 30))
        r = subprocess.run([plan_check, str(B), str(Hq), str(Hkv), str(T), str(C), "-1",
                            *map(str, lengths)], capture_output=True, text=True)
        assert r.returncode == 0, r.stdout


@pytest.mark.parametrize("window", [1, 64, 129, 512, 4096])
def test_sliding_window_plans(plan_check, window):
    # the attended range of every sequence and the per-row cut of every depth
    rng = np.random.default_rng(window)
    for _ in range(12):
        B = int(rng.integers(1, 5))
        T = int(rng.integers(1, min(window, 128) + 1))
        lengths = rng.integers(0, 5000, size=B)
        C = int(rng.integers(1, 12))
        env = dict(os.environ, PLAN_CHECK_WINDOW=str(window))
        r = subprocess.run([plan_check, str(B), "8", "2", str(T), str(C), "-1", *map(str, lengths)],
                           capture_output=True, text=True, env=env)
        assert r.returncode == 0, r.stdout


def _declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"LS_API\s+[\w\s\*]+?\b(ls_\w+)\s*\(", text)


def test_library_exports_every_declared_symbol(cuda_lib):
    names = _declared_symbols()
    from tree_verification_attention_longspec_b200.binding import EXPORTED
    assert set(EXPORTED) <= set(names)
    for n in names:
        assert hasattr(cuda_lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only",
                          os.path.join(ROOT, "tree_verification_attention_longspec_b200", "lib",
                                       "libls_verify_attn.so")], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (ls_\w+)", out))
    assert set(names) <= exported
    # nothing but the C-ABI is exported under the ls_ prefix
    assert exported == set(names)


def test_status_strings(cuda_lib):
    for code in range(8):
        s = cuda_lib.ls_status_string(code)
        assert s and s != b"unknown status"
    assert cuda_lib.ls_status_string(99) == b"unknown status"


def test_invalid_dims_rejected_on_host(cuda_lib):
    from tree_verification_attention_longspec_b200.binding import make_dims
    cases = [
        (dict(batch=1, num_q_heads=6, num_kv_heads=4, head_dim=128, tree_size=8), 1),
        (dict(batch=0, num_q_heads=4, num_kv_heads=4, head_dim=128, tree_size=8), 1),
        (dict(batch=1, num_q_heads=4, num_kv_heads=4, head_dim=96, tree_size=8), 2),
        (dict(batch=1, num_q_heads=4, num_kv_heads=4, head_dim=128, tree_size=129), 2),
        (dict(batch=1, num_q_heads=4, num_kv_heads=4, head_dim=128, tree_size=0), 1),
        (dict(batch=2, num_q_heads=4, num_kv_heads=4, head_dim=64, tree_size=4,
              cu_seqlens_host=[0, 10, 5]), 1),
        (dict(batch=2, num_q_heads=4, num_kv_heads=4, head_dim=64, tree_size=4,
              cu_seqlens_host=[1, 10, 15]), 1),
    ]
    for kw, want in cases:
        dims, keep = make_dims(**kw)
        rc = cuda_lib.ls_verify_attn(None, None, None, None, None, None, None, None, None,
                                     ctypes.byref(dims), None, 0, None)
        assert rc == want, (kw, rc)
        assert cuda_lib.ls_verify_attn_workspace_size(ctypes.byref(dims)) == 0


def test_binding_raises_when_library_missing(tmp_path):
    from tree_verification_attention_longspec_b200 import binding
    saved = binding._lib
    binding._lib = None
    try:
        with pytest.raises(RuntimeError, match="missing"):
            binding.load_library(str(tmp_path / "nope.so"))
    finally:
        binding._lib = saved
