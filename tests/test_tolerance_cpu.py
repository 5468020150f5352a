"""CPU checks of the error bound the GPU tests use for `out` (tests/gpu_harness.py).

The kernel rounds each softmax weight p_k to bf16 before the tensor-core PV product and
normalises by the sum of the rounded weights. The bound the tests assert for that step is
WEIGHT_ERR times the values' mean absolute deviation under the exact weights (at most
their weighted standard deviation). These checks replay exactly that arithmetic in fp64
(bf16 rounding to nearest even, nothing else) on random and adversarial weight sets and
verify the bound holds and is not loose by more than a small factor; and they check the
helper that gives the tests the values' weighted spread against the oracle.
"""
from __future__ import annotations

import numpy as np

from tests.gpu_harness import WEIGHT_ERR, value_spread
from tree_verification_attention_longspec_b200.inputs import Workload, bf16_bits_from_f32, bf16_bits_to_f64, make_inputs


def _rounded_average(p, v):
    """sum_k bf16(p_k) v_k / sum_k bf16(p_k), in fp64 after the rounding."""
    pr = bf16_bits_to_f64(bf16_bits_from_f32(p.astype(np.float32)))
    return (pr[:, None] * v).sum(axis=0) / pr.sum()


def _bound(p, v):
    w = p / p.sum()
    o = (w[:, None] * v).sum(axis=0)
    return o, WEIGHT_ERR * (w[:, None] * np.abs(v - o)).sum(axis=0)


def test_bound_holds_on_random_peaked_weights():
    rng = np.random.default_rng(0)
    worst = 0.0
    for _ in range(400):
        n = int(rng.integers(2, 600))
        scores = rng.standard_normal(n) * rng.choice([0.5, 2.0, 6.0, 12.0])
        p = np.exp2(scores - scores.max() + rng.uniform(0, 8))  # lazily rescaled: max in [1, 256)
        p = p.astype(np.float32).astype(np.float64)              # the kernel's fp32 weights
        v = rng.standard_normal((n, 8)) * rng.choice([1.0, 3.0, 10.0])
        o, b = _bound(p, v)
        err = np.abs(_rounded_average(p, v) - o)
        assert np.all(err <= b + 1e-12)
        worst = max(worst, float((err / np.maximum(b, 1e-300)).max()))
    assert worst > 0.05  # the bound is reached within a small factor on random sets


def test_bound_holds_and_is_nearly_reached_on_adversarial_weights():
    # half the keys weigh just above the midpoint 1 + 2^-8 between two bf16 numbers (they
    # round up by almost u = 2^-8) and carry the value +1, half just below it (they round
    # down by almost u) and carry -1: the rounding errors all push the average the same
    # way, and the error reaches about half the bound
    eps = 2.0 ** -16
    for n_half in (1, 4, 64):
        for e in (0, -3, 5):  # the same at other binades
            hi = np.full(n_half, (1.0 + 2.0 ** -8 + eps) * 2.0 ** e)
            lo = np.full(n_half, (1.0 + 2.0 ** -8 - eps) * 2.0 ** e)
            p = np.concatenate([hi, lo]).astype(np.float32).astype(np.float64)
            v = np.concatenate([np.ones(n_half), -np.ones(n_half)])[:, None]
            o, b = _bound(p, v)
            err = np.abs(_rounded_average(p, v) - o)
            assert np.all(err <= b)
            assert np.all(err >= 0.45 * b)


def test_value_spread_mean_is_the_oracle_output():
    import oracle
    w = Workload("spread", 2, 8, 2, 64, 16, 0, "window8", input_scale=2.0, lengths=[300, 129])
    inp = make_inputs(w, seed=3)
    mean, spread = value_spread(inp)
    ro, _ = oracle.verify_attn_oracle_inputs(inp)
    assert np.abs(mean - ro).max() < 1e-10
    assert np.all(spread >= 0) and np.all(np.isfinite(spread))
    # the spread of constant values is 0: all values equal -> the output equals them
    inp.v_cache[:] = bf16_bits_from_f32(np.float32([1.5]))[0]
    inp.v_tree[:] = bf16_bits_from_f32(np.float32([1.5]))[0]
    mean, spread = value_spread(inp)
    assert np.allclose(mean, 1.5) and spread.max() < 1e-7
