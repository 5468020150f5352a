"""GPU parity: the CUDA path through the C-ABI against the fp64 oracle on identical
seeded inputs. Tolerances: max-abs 1e-2 on bf16 `out`, 1e-3 on fp32 `lse`."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from tests.gpu_harness import LSE_ATOL, OUT_ATOL, make_op, out_tolerance, run_gpu, spread_tolerance, to_device, value_spread
from tree_verification_attention_longspec_b200.inputs import Workload, bf16_bits_to_f32, make_inputs
from tree_verification_attention_longspec_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu


def _compare(inp, out, lse, rows=None, scale=None):
    ro, rl = oracle.verify_attn_oracle_inputs(inp, rows=rows, scale=scale)
    if rows is not None:
        out, lse = out[rows], lse[rows]
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    err = np.abs(out - ro)
    excess = err - out_tolerance(ro)
    err_l = np.abs(lse - rl).max()
    assert excess.max() <= 0, (f"out error {err.flat[excess.argmax()]} at |ref| "
                               f"{abs(ro.flat[excess.argmax()])} (max-abs {err.max()})")
    assert err_l <= LSE_ATOL, f"lse max-abs {err_l}"
    return err.max(), err_l


def test_tiny_all_rows():
    inp = make_inputs(WORKLOADS["tiny_L1k_T16_h4x1_d64"], seed=0)
    out, lse, st = run_gpu(inp)
    assert st == 0
    _compare(inp, out, lse)


@pytest.mark.parametrize("name", ["llama8b_L16k_T64_h32x8_d128", "qwen7b_L64k_T64_h28x4_d128",
                                  "70b_L128k_T128_h64x8_d128_bfs", "ragged_b8_L4k-32k_T64_h32x8_d128"])
def test_full_size_all_rows(name):
    """Every output row of the full-size workloads against the oracle (seconds of fp64
    work per workload on the host cores), in the launch configuration bench.py times."""
    inp = make_inputs(WORKLOADS[name], seed=0)
    out, lse, st = run_gpu(inp)
    assert st == 0
    _compare(inp, out, lse)
    # properties of every row: finite; out is a convex combination of values, so it is
    # bounded by the largest |v|; lse is at least the score of the always-visible self key
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    vmax = max(np.abs(bf16_bits_to_f32(inp.v_cache)).max(), np.abs(bf16_bits_to_f32(inp.v_tree)).max())
    assert np.abs(out).max() <= vmax + OUT_ATOL
    w = inp.workload
    g = w.num_q_heads // w.num_kv_heads
    q = bf16_bits_to_f32(inp.q).astype(np.float64)                     # [B*T, Hq, d]
    kself = bf16_bits_to_f32(inp.k_tree).astype(np.float64)             # [B*T, Hkv, d]
    s_self = np.einsum("thd,thd->th", q, np.repeat(kself, g, axis=1)) * inp.scale
    assert np.all(lse >= s_self.reshape(-1) - LSE_ATOL)


def _small(B, Hq, Hkv, d, T, lengths, tree, seed=0, scale=1.0):
    w = Workload("edge", B, Hq, Hkv, d, T, 0, tree, input_scale=scale, lengths=lengths)
    return make_inputs(w, seed=seed)


EDGE = [
    # B, Hq, Hkv, d, T, lengths, tree
    (2, 4, 2, 128, 8, [0, 0], "uniform"),                 # empty prefix: tree only
    (3, 8, 2, 128, 16, [300, 129, 1], "window8"),          # ragged tails, not multiples of 128
    (2, 8, 8, 64, 1, [257, 1000], "chain"),                # T = 1: decode attention, MHA, d = 64
    (1, 4, 1, 128, 33, [700], "star"),                      # star tree
    (1, 4, 2, 64, 40, [512], "chain"),                      # chain tree = causal
    (1, 64, 8, 128, 128, [2000], "bfs"),                    # max tree, 1024 rows per kv head
    (1, 64, 1, 128, 4, [640], "uniform"),                   # group 64 (> warps per CTA)
    (5, 28, 4, 128, 64, [0, 1, 128, 4097, 2500], "window8"),
    (1, 2, 1, 64, 128, [3], "uniform"),
]


@pytest.mark.parametrize("B,Hq,Hkv,d,T,lengths,tree", EDGE)
def test_edge_cases_all_rows(B, Hq, Hkv, d, T, lengths, tree):
    inp = _small(B, Hq, Hkv, d, T, lengths, tree, seed=B * 7 + T)
    out, lse, st = run_gpu(inp)
    assert st == 0
    _compare(inp, out, lse)


MULTI_UNIT = [
    # d = 128 with two or four 256-row units per kv head, each unit above 128 rows (two
    # tiles, no alternate blocks). B, Hq, Hkv, T, lengths, tree
    (2, 14, 2, 64, [300, 1000], "window8"),   # g = 7: units of 252 and 196 rows, ragged tails
    (3, 16, 2, 64, [129, 0, 2049], "bfs"),    # g = 8: two full units; an empty prefix
    (1, 32, 4, 128, [777], "chain"),          # g = 8, T = 128: four units per kv head
]


@pytest.mark.parametrize("B,Hq,Hkv,T,lengths,tree", MULTI_UNIT)
@pytest.mark.parametrize("host_lengths", [True, False])
def test_multi_unit_kv_heads_all_rows(B, Hq, Hkv, T, lengths, tree, host_lengths):
    inp = _small(B, Hq, Hkv, 128, T, lengths, tree, seed=B * 11 + T)
    out, lse, st = run_gpu(inp, host_lengths=host_lengths)
    assert st == 0
    _compare(inp, out, lse)


def test_large_batch_with_host_lengths():
    # more sequences than the plan carries host lengths for (32): the kernels read the
    # device cu_seqlens, with per-sequence chunk counts from the host copy
    rng = np.random.default_rng(9)
    lengths = [int(x) for x in rng.integers(0, 700, size=40)]
    inp = _small(40, 8, 2, 64, 6, lengths, "uniform", seed=9)
    out, lse, st = run_gpu(inp)
    assert st == 0
    _compare(inp, out, lse)


def test_uniform_plan_without_host_lengths():
    inp = _small(4, 16, 4, 128, 12, [5000, 0, 130, 2049], "uniform", seed=3)
    out, lse, st = run_gpu(inp, host_lengths=False)
    assert st == 0
    _compare(inp, out, lse)


def test_custom_softmax_scale():
    inp = _small(2, 8, 2, 128, 10, [333, 1024], "window8", seed=4)
    out, lse, st = run_gpu(inp, scale=0.05)
    assert st == 0
    _compare(inp, out, lse, scale=0.05)


def test_repeat_calls_are_bitwise_identical():
    inp = _small(2, 28, 4, 128, 64, [3000, 9000], "window8", seed=5)
    dev = to_device(inp)
    op = make_op(inp)
    o1, l1, s1 = run_gpu(inp, dev=dev, op=op)
    o2, l2, s2 = run_gpu(inp, dev=dev, op=op)
    assert s1 == s2 == 0
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_bad_tree_reported():
    inp = _small(2, 4, 2, 128, 8, [200, 300], "uniform", seed=6)
    inp.parent[8 + 5] = 6          # parent after child in sequence 1
    _, _, st = run_gpu(inp)
    assert st == 5                  # LS_ERR_BAD_TREE
    inp = _small(1, 4, 2, 128, 8, [200], "uniform", seed=6)
    inp.parent[0] = 0               # root with a parent
    _, _, st = run_gpu(inp)
    assert st == 5


def test_length_mismatch_reported():
    """The host copy of cu_seqlens disagrees with the device array: the call must stay
    in bounds and report LS_ERR_LENGTHS."""
    import torch
    inp = _small(2, 8, 2, 128, 8, [1000, 3000], "uniform", seed=7)
    dev = to_device(inp)
    op = make_op(inp)
    short = inp.cu_seqlens.copy()
    short[2] = 1000 + 200           # device says sequence 1 is shorter than planned
    dev["cu_seqlens"] = torch.from_numpy(short).to("cuda:0")
    _, _, st = run_gpu(inp, dev=dev, op=op)
    assert st == 7                  # LS_ERR_LENGTHS


def test_workspace_contents_do_not_matter():
    """The workspace needs no initialisation: NaN bytes in it (including the slots of
    empty chunks, which are never written) must not reach the output."""
    inp = _small(4, 8, 2, 128, 10, [700, 0, 1, 3000], "uniform", seed=8)
    dev = to_device(inp)
    op = make_op(inp, host_lengths=False)
    op.workspace.fill_(0xFF)
    out, lse, st = run_gpu(inp, dev=dev, op=op)
    assert st == 0
    _compare(inp, out, lse)


@pytest.mark.parametrize("scale", [2.0, 3.0])
def test_peaked_softmax_all_rows(scale):
    """Inputs drawn N(0, scale^2), beyond the workloads' N(0, 1): the scores' spread grows
    as scale^2 (std 4 and 9), so rows are dominated by a few keys, the running max is
    raised well past the lazy threshold as the blocks go by, and the weights' bf16
    rounding does not average out. The values spread as widely (std scale), and a fixed
    1e-2 no longer holds: the bound is the one the weights' rounding gives, half an ulp
    plus 2^-7 of the values' weighted spread (gpu_harness.spread_tolerance)."""
    inp = _small(2, 28, 4, 128, 64, [3000, 9000], "window8", seed=int(scale * 10), scale=scale)
    out, lse, st = run_gpu(inp)
    assert st == 0
    ro, rl = oracle.verify_attn_oracle_inputs(inp)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    mean, spread = value_spread(inp)
    assert np.abs(mean - ro).max() < 1e-9  # the helper's weights are the oracle's
    tol = spread_tolerance(ro, spread)
    err = np.abs(out - ro)
    assert np.all(err <= tol), f"out error {err.flat[(err - tol).argmax()]} over {tol.flat[(err - tol).argmax()]}"
    assert np.abs(lse - rl).max() <= LSE_ATOL


def test_keys_growing_along_the_sequence_all_rows():
    """Key vectors scaled by a ramp from 0.25 to 3 along each sequence: every block tends
    to raise the running max of its rows, so the O rescale runs block after block."""
    from tree_verification_attention_longspec_b200.inputs import bf16_bits_from_f32, bf16_bits_to_f32
    inp = _small(2, 16, 2, 128, 32, [5000, 2500], "bfs", seed=44)
    k = bf16_bits_to_f32(inp.k_cache)
    for b in range(2):
        s0, s1 = int(inp.cu_seqlens[b]), int(inp.cu_seqlens[b + 1])
        ramp = np.linspace(0.25, 3.0, s1 - s0, dtype=np.float32)[:, None, None]
        k[s0:s1] *= ramp
    inp.k_cache = bf16_bits_from_f32(k)
    out, lse, st = run_gpu(inp)
    assert st == 0
    _compare(inp, out, lse)


@pytest.mark.parametrize("host_lengths", [True, False])
def test_group_256_one_node_per_unit(host_lengths):
    # g = 256, the largest group: a unit holds one tree node's 256 heads
    inp = _small(2, 256, 1, 64, 3, [700, 129], "chain", seed=45)
    out, lse, st = run_gpu(inp, host_lengths=host_lengths)
    assert st == 0
    _compare(inp, out, lse)


@pytest.mark.parametrize("B", [32, 33])
def test_batch_at_the_plan_s_host_length_limit(B):
    # the plan carries host lengths for B <= 32 and reads the device array beyond
    rng = np.random.default_rng(B)
    lengths = [int(x) for x in rng.integers(0, 1500, size=B)]
    inp = _small(B, 8, 2, 128, 4, lengths, "uniform", seed=B)
    out, lse, st = run_gpu(inp)
    assert st == 0
    _compare(inp, out, lse)
