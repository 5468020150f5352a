"""ls_verify_attn_static: the entry point for callers that cannot allocate device memory.

Some callers only hold their input and output buffers, for example an operator plugin
inside an inference engine that owns all device memory and gives its plugins no
allocator. They cannot pass the workspace that ls_verify_attn needs, so
ls_verify_attn_static uses scratch that lives in the library itself. These checks call
it through the C-ABI and compare it with the regular entry point on the same inputs.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

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


def test_static_scratch_matches_workspace_call():
    w = Workload("no_alloc", batch=2, num_q_heads=28, num_kv_heads=4, head_dim=128, tree_size=64, prefix=0,
                 tree="window8", lengths=[3000, 9100])
    inp = make_inputs(w, seed=21)
    dev = to_device(inp)
    op = make_op(inp)
    assert op.ws_bytes <= STATIC_SCRATCH_BYTES
    ref_out, ref_lse = op(dev["q"], dev["k_cache"], dev["v_cache"], dev["k_tree"], dev["v_tree"], dev["parent"],
                          dev["cu_seqlens"])
    torch.cuda.synchronize()
    assert op.check() == 0
    ref_o = ref_out.float().cpu().numpy().astype(np.float64)
    ref_l = ref_lse.cpu().numpy().astype(np.float64)
    for _ in range(2):  # two calls in a row share (and reuse) the library's scratch
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        assert _static_call(dev, op.dims, out, lse) == binding.LS_OK
        torch.cuda.synchronize()
        o = out.float().cpu().numpy().astype(np.float64)
        l_ = lse.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(l_))
        assert np.all(np.abs(o - ref_o) <= out_tolerance(ref_o))
        assert np.abs(l_ - ref_l).max() <= LSE_ATOL


def test_static_scratch_rejects_dims_beyond_its_size():
    dims, _keep = binding.make_dims(batch=1, num_q_heads=64, num_kv_heads=8, head_dim=128, tree_size=128,
                                    max_prefix_len=131072)
    assert binding.workspace_size(dims) > STATIC_SCRATCH_BYTES
    lib = binding.load_library()
    rc = lib.ls_verify_attn_static(None, None, None, None, None, None, None, None, None, ctypes.byref(dims), None)
    assert rc == 3  # LS_ERR_WORKSPACE, before anything is launched
