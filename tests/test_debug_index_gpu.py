"""The index-checking build (libls_verify_attn_debug.so, LS_DEBUG) on the GPU.

The same sources compiled with LS_DEBUG check every TMA coordinate and global index the
kernels form against the extent of the tensor it addresses: the unmasked rows of each
K/V box lie inside their sequence and the cache, each page box of a paged cache comes
from a page-table entry inside the pages, the tree and Q boxes inside the tree tensors,
every partial the combine reads inside the workspace, every output row inside out/lse.
A failed check is reported as LS_ERR_INDEX by ls_verify_attn_check. These checks run the
small cases of the other GPU tests through that library: none may report a violation,
and the results must still match the oracle. One case plants a page-table entry outside
the pages (the release library accepts it as documented, reading zeros there) to show
that the checks are live.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_harness import LSE_ATOL, out_tolerance, to_device
from tests.test_paged_gpu import _paged
from tree_verification_attention_longspec_b200 import binding, build
from tree_verification_attention_longspec_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu

LS_ERR_INDEX = 8


@pytest.fixture(scope="module")
def dlib():
    build.build(debug=True)
    return binding.load_debug_library()


def _dims(inp, host_lengths=True):
    w = inp.workload
    L = np.diff(inp.cu_seqlens)
    return binding.make_dims(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.tree_size,
                             max_prefix_len=int(L.max()) if len(L) else 0,
                             cu_seqlens_host=inp.cu_seqlens if host_lengths else None)


def _run(dlib, inp, host_lengths=True, page=None, tree=None, cross=False):
    """One call through the debug library; returns (out, lse, status) as float64 arrays."""
    w = inp.workload
    dev = to_device(inp)
    dims, keep = _dims(inp, host_lengths)
    t_ref = None if tree is None else ctypes.byref(tree)
    if cross:
        wsb = int(dlib.ls_cross_attn_workspace_size(ctypes.byref(dims)))
    else:
        wsb = int(dlib.ls_verify_attn_ex_workspace_size(ctypes.byref(dims), t_ref))
    assert wsb > 0
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    out = torch.full_like(dev["q"], float("nan"))
    lse = torch.full((out.shape[0], w.num_q_heads), float("nan"), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    kc, vc = dev["k_cache"].data_ptr(), dev["v_cache"].data_ptr()
    pg = None
    if page is not None:
        kc, vc, pg, keep_pages = page
    if cross:
        rc = dlib.ls_cross_attn(dev["q"].data_ptr(), kc, vc, dev["cu_seqlens"].data_ptr(), out.data_ptr(),
                                lse.data_ptr(), ctypes.byref(dims), ws.data_ptr(), wsb, stream)
    else:
        rc = dlib.ls_verify_attn_ex(dev["q"].data_ptr(), kc, vc, None if pg is None else ctypes.byref(pg),
                                    dev["k_tree"].data_ptr(), dev["v_tree"].data_ptr(), dev["parent"].data_ptr(),
                                    dev["cu_seqlens"].data_ptr(), t_ref, out.data_ptr(), lse.data_ptr(),
                                    ctypes.byref(dims), ws.data_ptr(), wsb, stream)
    assert rc == binding.LS_OK, binding.STATUS_NAMES.get(rc, rc)
    torch.cuda.synchronize()
    st = int(dlib.ls_verify_attn_check(ctypes.byref(dims), ws.data_ptr(), stream))
    o = out.float().cpu().numpy().astype(np.float64).reshape(-1, w.head_dim)
    l_ = lse.cpu().numpy().astype(np.float64).reshape(-1)
    return o, l_, st


def _close(o, l_, ro, rl):
    assert np.all(np.abs(o - ro) <= out_tolerance(ro))
    assert np.abs(l_ - rl).max() <= LSE_ATOL


def _pages(inp, page_size, bad_entry=False):
    kp, vp, table, num_pages = _paged(inp, page_size)
    if bad_entry:
        table = table.copy()
        table[0, 0] = num_pages + 5  # a page that holds keys, outside the pages
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)  # noqa: E731
    kd, vd, td = bf(kp), bf(vp), torch.from_numpy(table).cuda()
    pg = binding.PagedKV(page_size, table.shape[1], num_pages, td.data_ptr())
    return kd.data_ptr(), vd.data_ptr(), pg, (kd, vd, td)


CASES = [
    # B, Hq, Hkv, d, T, lengths, tree, host lengths
    (1, 4, 1, 64, 16, [1024], "uniform", True),                 # the tiny workload's shape
    (2, 4, 2, 128, 8, [0, 0], "uniform", True),                  # tree only
    (3, 8, 2, 128, 16, [300, 129, 1], "window8", True),         # ragged tails
    (5, 28, 4, 128, 64, [0, 1, 128, 4097, 2500], "window8", True),
    (1, 64, 8, 128, 128, [2000], "bfs", True),                   # four units per kv head
    (1, 64, 1, 128, 4, [640], "uniform", True),                  # group 64
    (4, 16, 4, 128, 12, [5000, 0, 130, 2049], "uniform", False),  # uniform plan, device lengths
]


@pytest.mark.parametrize("B,Hq,Hkv,d,T,lengths,tree,host", CASES)
def test_no_index_violation(dlib, B, Hq, Hkv, d, T, lengths, tree, host):
    inp = make_inputs(Workload("dbg", B, Hq, Hkv, d, T, 0, tree, input_scale=1.0, lengths=lengths), seed=B + T)
    o, l_, st = _run(dlib, inp, host_lengths=host)
    assert st == binding.LS_OK, binding.STATUS_NAMES.get(st, st)
    ro, rl = oracle.verify_attn_oracle_inputs(inp)
    _close(o, l_, ro, rl)


@pytest.mark.parametrize("page_size", [16, 64, 256])
def test_paged_no_index_violation(dlib, page_size):
    inp = make_inputs(Workload("dbg_paged", 4, 8, 2, 128, 16, 0, "uniform", input_scale=1.0,
                               lengths=[1000, 0, 2500, 9]), seed=3)
    page = _pages(inp, page_size)
    o, l_, st = _run(dlib, inp, page=page)
    assert st == binding.LS_OK, binding.STATUS_NAMES.get(st, st)
    ro, rl = oracle.verify_attn_oracle_inputs(inp)
    _close(o, l_, ro, rl)


def test_ragged_trees_rope_window_no_index_violation(dlib):
    from oracle import tree_positions as tp
    w = Workload("dbg_ex", 3, 16, 4, 128, 96, 0, "bfs", lengths=[700, 1, 2100], tree_sizes=[96, 40, 3])
    inp = make_inputs(w, seed=24)
    cu_tree = torch.from_numpy(inp.cu_tree.astype(np.int32)).cuda()
    theta, window = 500000.0, 600
    tree = binding.TreeOpts(cu_tree=cu_tree.data_ptr(), total_nodes=inp.num_nodes, window=window,
                            rope_theta=theta)
    o, l_, st = _run(dlib, inp, tree=tree, page=_pages(inp, 16))
    assert st == binding.LS_OK, binding.STATUS_NAMES.get(st, st)
    pos = tp.tree_positions(inp.parent, inp.cu_seqlens, inp.node_offsets())
    qr, kr = tp.rope_bf16(inp.q, pos, theta), tp.rope_bf16(inp.k_tree, pos, theta)
    ro, rl = oracle.verify_attn_oracle_window(qr, inp.k_cache, inp.v_cache, kr, inp.v_tree, inp.parent,
                                              inp.cu_seqlens, inp.node_offsets(), num_q_heads=16, num_kv_heads=4,
                                              head_dim=128, scale=inp.scale, window=window)
    _close(o, l_, ro, rl)


def test_cross_attention_no_index_violation(dlib):
    from tests.test_cross_gpu import _oracle_rows
    inp = make_inputs(Workload("dbg_cross", 3, 8, 2, 64, 4, 0, "chain", input_scale=1.0,
                               lengths=[333, 0, 1500]), seed=12)
    o, l_, st = _run(dlib, inp, cross=True)
    assert st == binding.LS_OK, binding.STATUS_NAMES.get(st, st)
    w = inp.workload
    empty = np.repeat(np.diff(inp.cu_seqlens) == 0, w.tree_size * w.num_q_heads)
    assert np.all(o[empty] == 0) and np.all(np.isneginf(l_[empty]))
    rows = np.flatnonzero(~empty)
    ro, rl = _oracle_rows(inp, rows)
    _close(o[rows], l_[rows], ro, rl)


def test_planted_page_outside_the_pages_is_reported(dlib):
    """A page-table entry outside the pages for a page that holds keys: the release build
    documents it as reading zeros (no fault, unspecified result); the checking build
    reports it."""
    inp = make_inputs(Workload("dbg_bad", 2, 8, 2, 128, 8, 0, "uniform", input_scale=1.0, lengths=[700, 300]),
                      seed=5)
    _, _, st = _run(dlib, inp, page=_pages(inp, 64, bad_entry=True))
    assert st == LS_ERR_INDEX
    _, _, st = _run(dlib, inp, page=_pages(inp, 64))
    assert st == binding.LS_OK
