"""The stall detector of the partials kernel, driven to expiry.

Every device-side wait of the partials kernel (a CTA's TMA producer, MMA thread and
softmax warps hand tiles to one another through shared-memory barriers) is bounded by
the call's wait limit, ls_tree_opts.wait_limit_ns (4 s by default). These checks set the
limit to one nanosecond, far shorter than the normal waits of a healthy call, so that
waits run out, and verify what a stalled call must do: return, report LS_ERR_TIMEOUT
through ls_verify_attn_check, and leave nothing behind, so that the next call on the same
stream and workspace gives bit for bit what a call on a fresh workspace gives.

Nothing here faults or hangs the GPU: a wait that runs out only stops its CTA early; the
copies and tensor-core work that were already issued still complete, and each CTA drains
them before it frees its tensor memory and returns.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_harness import LSE_ATOL, out_tolerance, to_device
from tests.test_paged_gpu import _paged
from tree_verification_attention_longspec_b200 import binding
from tree_verification_attention_longspec_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu

LS_ERR_TIMEOUT = 6


class _Call:
    """One problem on the device: runs ls_verify_attn_ex with or without a wait limit."""

    def __init__(self, inp, page_size=None):
        w = inp.workload
        self.inp = inp
        self.dev = to_device(inp)
        self.dims, self._keep = binding.make_dims(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.tree_size,
                                                  cu_seqlens_host=inp.cu_seqlens)
        self.kc, self.vc = self.dev["k_cache"].data_ptr(), self.dev["v_cache"].data_ptr()
        self.paged = None
        if page_size is not None:
            kp, vp, table, num_pages = _paged(inp, page_size)

            def bf(a):
                return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)

            self._pages = (bf(kp), bf(vp), torch.from_numpy(table).cuda())
            self.paged = binding.PagedKV(page_size, table.shape[1], num_pages, self._pages[2].data_ptr())
            self.kc, self.vc = self._pages[0].data_ptr(), self._pages[1].data_ptr()
        self.wsb = binding.ex_workspace_size(self.dims, binding.TreeOpts())
        assert self.wsb > 0
        self.stream = torch.cuda.current_stream().cuda_stream

    def new_workspace(self):
        return torch.empty(self.wsb, dtype=torch.uint8, device="cuda")

    def run(self, ws, wait_limit_ns=0):
        """Returns (out bf16 bits, lse fp32 bits, device status) of one call."""
        d = self.dev
        tree = binding.TreeOpts(wait_limit_ns=wait_limit_ns)
        out = torch.full_like(d["q"], float("nan"))
        lse = torch.full((out.shape[0], self.inp.workload.num_q_heads), float("nan"), dtype=torch.float32,
                         device="cuda")
        rc = binding.call_ex_raw(d["q"].data_ptr(), self.kc, self.vc, self.paged, d["k_tree"].data_ptr(),
                                 d["v_tree"].data_ptr(), d["parent"].data_ptr(), d["cu_seqlens"].data_ptr(), tree,
                                 out.data_ptr(), lse.data_ptr(), self.dims, ws.data_ptr(), self.wsb, self.stream)
        assert rc == binding.LS_OK, binding.STATUS_NAMES.get(rc, rc)
        torch.cuda.synchronize()
        status = binding.check(self.dims, ws.data_ptr(), self.stream)
        return out.view(torch.int16).cpu().numpy(), lse.view(torch.int32).cpu().numpy(), status


CASES = [
    # B, Hq, Hkv, d, T, lengths, tree, page size
    (2, 28, 4, 128, 64, [9000, 20000], "window8", None),   # g = 7: two 128-row tiles per unit
    (1, 4, 1, 64, 16, [30000], "uniform", None),            # 64 rows: alternate-block mode, d = 64
    (2, 16, 2, 128, 24, [5000, 12000], "bfs", 16),          # paged cache: the producer's page boxes
]


@pytest.mark.parametrize("B,Hq,Hkv,d,T,lengths,tree,page_size", CASES)
def test_expired_waits_are_reported_and_leave_nothing_behind(B, Hq, Hkv, d, T, lengths, tree, page_size):
    w = Workload("timeout", B, Hq, Hkv, d, T, 0, tree, input_scale=1.0, lengths=lengths)
    inp = make_inputs(w, seed=31 + d + T)
    call = _Call(inp, page_size)
    ws = call.new_workspace()
    # three stalled calls in a row on one workspace: each returns and reports the timeout
    for _ in range(3):
        _, _, st = call.run(ws, wait_limit_ns=1)
        assert st == LS_ERR_TIMEOUT
    # the next healthy call on the same stream and workspace: exact and clean
    o1, l1, st1 = call.run(ws)
    assert st1 == binding.LS_OK
    o2, l2, st2 = call.run(call.new_workspace())
    assert st2 == binding.LS_OK
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    # and it is the attention the oracle computes
    out = torch.from_numpy(o1).view(torch.bfloat16).float().numpy().astype(np.float64).reshape(-1, d)
    lse = l1.view(np.float32).astype(np.float64).reshape(-1)
    ro, rl = oracle.verify_attn_oracle_inputs(inp)
    assert np.all(np.abs(out - ro) <= out_tolerance(ro))
    assert np.abs(lse - rl).max() <= LSE_ATOL


def test_a_generous_limit_changes_nothing():
    w = Workload("timeout", 1, 28, 4, 128, 64, 0, "window8", input_scale=1.0, lengths=[7000])
    call = _Call(make_inputs(w, seed=40))
    o1, l1, s1 = call.run(call.new_workspace())                          # default: 4 s
    o2, l2, s2 = call.run(call.new_workspace(), wait_limit_ns=10 ** 9)   # 1 s
    assert s1 == s2 == binding.LS_OK
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_limit_above_a_minute_is_rejected_on_the_host():
    w = Workload("timeout", 1, 4, 1, 64, 8, 0, "uniform", input_scale=1.0, lengths=[500])
    call = _Call(make_inputs(w, seed=41))
    assert binding.ex_workspace_size(call.dims, binding.TreeOpts(wait_limit_ns=61 * 10 ** 9)) == 0
    assert binding.ex_workspace_size(call.dims, binding.TreeOpts(wait_limit_ns=60 * 10 ** 9)) > 0
