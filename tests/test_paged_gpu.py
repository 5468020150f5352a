"""GPU parity of the paged K/V cache entry point (ls_verify_attn_paged) against the fp64
oracle: the same seeded inputs as the packed path, with the prefix keys scattered into
randomly permuted pages. Pages past a sequence's end are filled with garbage and the
table columns past its last page with out-of-range entries, so that reading either would
show up as an error."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_harness import LSE_ATOL, make_op, out_tolerance, to_device
from tree_verification_attention_longspec_b200 import binding
from tree_verification_attention_longspec_b200.inputs import Workload, make_inputs
from tree_verification_attention_longspec_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu


def _paged(inp, page_size, seed=5, spare=3):
    """Scatter k_cache / v_cache into pages. Returns (k_pages, v_pages, table, num_pages)."""
    w = inp.workload
    cu = inp.cu_seqlens
    L = np.diff(cu)
    n_pages = [(int(x) + page_size - 1) // page_size for x in L]
    total = sum(n_pages) + spare
    rng = np.random.default_rng(seed)
    perm = rng.permutation(total)
    row_shape = inp.k_cache.shape[1:]
    # garbage everywhere (finite, large), then the real rows
    kp = rng.integers(0x4000, 0x4400, size=(total * page_size,) + row_shape).astype(np.uint16)
    vp = rng.integers(0x4000, 0x4400, size=(total * page_size,) + row_shape).astype(np.uint16)
    max_pages = max(max(n_pages), 1) + 2
    table = np.full((w.batch, max_pages), 1 << 28, dtype=np.int32)  # never read
    nxt = 0
    for b in range(w.batch):
        for i in range(n_pages[b]):
            phys = int(perm[nxt])
            nxt += 1
            table[b, i] = phys
            k0, k1 = cu[b] + i * page_size, min(cu[b] + (i + 1) * page_size, cu[b + 1])
            kp[phys * page_size: phys * page_size + (k1 - k0)] = inp.k_cache[k0:k1]
            vp[phys * page_size: phys * page_size + (k1 - k0)] = inp.v_cache[k0:k1]
    return kp, vp, table, total


def _run_paged(inp, page_size):
    w = inp.workload
    kp, vp, table, num_pages = _paged(inp, page_size)
    dev = to_device(inp)

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)

    kp_d, vp_d = bf(kp), bf(vp)
    tab_d = torch.from_numpy(table).cuda()
    op = make_op(inp)
    pg = binding.PagedKV(page_size, table.shape[1], num_pages, tab_d.data_ptr())
    out = torch.empty_like(dev["q"])
    lse = torch.empty(out.shape[0], w.num_q_heads, dtype=torch.float32, device="cuda")
    rc = binding.call_paged_raw(dev["q"].data_ptr(), kp_d.data_ptr(), vp_d.data_ptr(), pg, dev["k_tree"].data_ptr(),
                                dev["v_tree"].data_ptr(), dev["parent"].data_ptr(), dev["cu_seqlens"].data_ptr(),
                                out.data_ptr(), lse.data_ptr(), op.dims, op.workspace.data_ptr(), op.ws_bytes,
                                torch.cuda.current_stream().cuda_stream)
    assert rc == binding.LS_OK
    torch.cuda.synchronize()
    assert op.check() == 0
    o = out.float().cpu().numpy().astype(np.float64).reshape(-1, w.head_dim)
    l_ = lse.cpu().numpy().astype(np.float64).reshape(-1)
    return o, l_


def _check(inp, o, l_, rows=None):
    ro, rl = oracle.verify_attn_oracle_inputs(inp, rows=rows)
    if rows is not None:
        o, l_ = o[rows], l_[rows]
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(l_))
    assert np.all(np.abs(o - ro) <= out_tolerance(ro)), np.abs(o - ro).max()
    assert np.abs(l_ - rl).max() <= LSE_ATOL


@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("d", [64, 128])
def test_paged_small_all_rows(page_size, d):
    # lengths off every page and block boundary, an empty sequence, one shorter than a page
    w = Workload("paged", 4, 8, 2, d, 16, 0, "uniform", input_scale=1.0, lengths=[1000, 0, 2500, 9])
    inp = make_inputs(w, seed=3)
    o, l_ = _run_paged(inp, page_size)
    _check(inp, o, l_)


@pytest.mark.parametrize("page_size", [16, 64])
def test_paged_two_tile_units_all_rows(page_size):
    # 192 rows per kv head (g = 8, T = 24): a unit of two 128-row tiles, not alternating
    w = Workload("paged2t", 3, 16, 2, 128, 24, 0, "bfs", input_scale=1.0, lengths=[777, 3000, 130])
    inp = make_inputs(w, seed=4)
    o, l_ = _run_paged(inp, page_size)
    _check(inp, o, l_)


@pytest.mark.parametrize("page_size", [16, 128])
def test_paged_headline_all_rows(page_size):
    inp = make_inputs(WORKLOADS["qwen7b_L64k_T64_h28x4_d128"], seed=0)
    o, l_ = _run_paged(inp, page_size)
    _check(inp, o, l_)


def test_paged_rejects_bad_page_sizes():
    inp = make_inputs(WORKLOADS["tiny_L1k_T16_h4x1_d64"], seed=0)
    op = make_op(inp)
    dev = to_device(inp)
    for ps, maxp, want in ((48, 64, 2), (8, 256, 2), (192, 16, 2), (16, 10, 1)):  # 1024 keys need 64 pages of 16
        tab = torch.zeros(maxp, dtype=torch.int32, device="cuda")
        pg = binding.PagedKV(ps, maxp, 64, tab.data_ptr())
        rc = binding.call_paged_raw(dev["q"].data_ptr(), dev["k_cache"].data_ptr(), dev["v_cache"].data_ptr(), pg,
                                    dev["k_tree"].data_ptr(), dev["v_tree"].data_ptr(), dev["parent"].data_ptr(),
                                    dev["cu_seqlens"].data_ptr(), dev["q"].data_ptr(), dev["q"].data_ptr(), op.dims,
                                    op.workspace.data_ptr(), op.ws_bytes, 0)
        assert rc == want, (ps, maxp, rc)
