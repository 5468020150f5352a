"""ls_verify_attn_static: the entry point for callers that cannot allocate device memory.

Some callers only hold their input and output buffers, for example an operator plugin
inside an inference engine that owns all device memory and gives its plugins no
allocator. They cannot pass the workspace that ls_verify_attn needs, so
ls_verify_attn_static uses scratch that lives in the library itself. These checks call
it through the C-ABI and compare it with the regular entry point on the same inputs and
with the fp64 oracle, over calls of different sizes that reuse the shared scratch.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_harness import LSE_ATOL, make_op, out_tolerance, to_device
from tree_verification_attention_longspec_b200 import binding
from tree_verification_attention_longspec_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 32 << 20


def _static_call(dev, dims, out, lse):
    stream = torch.cuda.current_stream()
    return binding.call_static_raw(dev["q"].data_ptr(), dev["k_cache"].data_ptr(), dev["v_cache"].data_ptr(),
                                   dev["k_tree"].data_ptr(), dev["v_tree"].data_ptr(), dev["parent"].data_ptr(),
                                   dev["cu_seqlens"].data_ptr(), out.data_ptr(), lse.data_ptr(), dims,
                                   stream.cuda_stream)


def _to_np(out, lse):
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


class _Problem:
    """Inputs on the device, the workspace call's result and the oracle's."""

    def __init__(self, w, seed, host_lengths):
        self.inp = make_inputs(w, seed=seed)
        self.dev = to_device(self.inp)
        self.op = make_op(self.inp, host_lengths=host_lengths)
        d = self.dev
        ref_out, ref_lse = self.op(d["q"], d["k_cache"], d["v_cache"], d["k_tree"], d["v_tree"], d["parent"],
                                   d["cu_seqlens"])
        torch.cuda.synchronize()
        assert self.op.check() == 0
        self.like = (ref_out, ref_lse)
        self.ref = _to_np(ref_out, ref_lse)
        ro, rl = oracle.verify_attn_oracle_inputs(self.inp)
        self.oracle = (ro.reshape(self.ref[0].shape), rl.reshape(self.ref[1].shape))

    def static_call_matches(self):
        out = torch.full_like(self.like[0], float("nan"))
        lse = torch.full_like(self.like[1], float("nan"))
        assert _static_call(self.dev, self.op.dims, out, lse) == binding.LS_OK
        torch.cuda.synchronize()
        o, l_ = _to_np(out, lse)
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(l_))
        for ref_o, ref_l in (self.ref, self.oracle):
            assert np.all(np.abs(o - ref_o) <= out_tolerance(ref_o))
            assert np.abs(l_ - ref_l).max() <= LSE_ATOL


LARGE = Workload("no_alloc", batch=2, num_q_heads=28, num_kv_heads=4, head_dim=128, tree_size=64, prefix=0,
                 tree="window8", lengths=[3000, 9100])
SMALL = Workload("no_alloc_small", batch=1, num_q_heads=4, num_kv_heads=1, head_dim=64, tree_size=16, prefix=0,
                 tree="uniform", input_scale=1.0, lengths=[1000])


@pytest.mark.parametrize("host_lengths", [True, False])
def test_static_scratch_matches_workspace_call(host_lengths):
    """Two calls in a row share (and reuse) the library's scratch; with host lengths the
    plan is balanced on the actual lengths, without them on max_prefix_len."""
    prob = _Problem(LARGE, seed=21, host_lengths=host_lengths)
    assert bool(prob.op.dims.cu_seqlens_host) == host_lengths
    assert prob.op.ws_bytes <= STATIC_SCRATCH_BYTES
    for _ in range(2):
        prob.static_call_matches()


def test_large_then_small_call_leaves_no_stale_partials():
    """A call that fills most of the scratch, then one that needs a fraction of it, then
    the large one again: each matches its own workspace call and the oracle."""
    large = _Problem(LARGE, seed=22, host_lengths=True)
    small = _Problem(SMALL, seed=23, host_lengths=True)
    assert small.op.ws_bytes * 8 < large.op.ws_bytes <= STATIC_SCRATCH_BYTES
    large.static_call_matches()
    small.static_call_matches()
    large.static_call_matches()


def test_static_scratch_rejects_dims_beyond_its_size():
    # 32 sequences of a 70B-shaped layer: over a thousand 256-row chunk partials
    dims, _keep = binding.make_dims(batch=32, num_q_heads=64, num_kv_heads=8, head_dim=128, tree_size=128,
                                    max_prefix_len=131072)
    assert binding.workspace_size(dims) > STATIC_SCRATCH_BYTES
    lib = binding.load_library()
    rc = lib.ls_verify_attn_static(None, None, None, None, None, None, None, None, None, ctypes.byref(dims), None)
    assert rc == 3  # LS_ERR_WORKSPACE, before anything is launched
