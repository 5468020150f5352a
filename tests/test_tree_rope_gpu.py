"""GPU parity of ls_verify_attn_ex — per-sequence trees (cu_tree) and in-kernel RoPE at
tree positions — against the fp64 oracle. The oracle rotates q and k_tree at positions
L_b + depth(i) (oracle/tree_positions.py), rounds them to bf16 and runs the plain
softmax of each sequence over its prefix and its ancestor-or-self tree nodes."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle import tree_positions as tp
from tests.gpu_harness import LSE_ATOL, out_tolerance, to_device
from tests.test_paged_gpu import _paged
from tree_verification_attention_longspec_b200 import binding
from tree_verification_attention_longspec_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu


def _tree_opts(inp, theta, cu_tree_dev, window=0):
    if inp.cu_tree is None and theta == 0.0 and window == 0:
        return None
    ragged = inp.cu_tree is not None
    return binding.TreeOpts(cu_tree=cu_tree_dev.data_ptr() if ragged else None,
                            total_nodes=inp.num_nodes if ragged else 0, window=window, rope_theta=float(theta))


def _run_ex(inp, theta=0.0, page_size=None, host_lengths=True, cu_tree_dev=None, expect_rc=binding.LS_OK,
            window=0):
    """Returns (out fp64 [N*H_q, d], lse fp64 [N*H_q], device status, q after the call)."""
    w = inp.workload
    dev = to_device(inp)
    L = np.diff(inp.cu_seqlens)
    dims, keep = binding.make_dims(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.tree_size,
                                   max_prefix_len=int(L.max()) if len(L) else 0,
                                   cu_seqlens_host=inp.cu_seqlens if host_lengths else None)
    if cu_tree_dev is None and inp.cu_tree is not None:
        cu_tree_dev = torch.from_numpy(inp.cu_tree.astype(np.int32)).cuda()
    tree = _tree_opts(inp, theta, cu_tree_dev, window)
    wsb = binding.ex_workspace_size(dims, tree)
    assert wsb > 0
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    out = torch.full_like(dev["q"], float("nan"))
    lse = torch.full((out.shape[0], w.num_q_heads), float("nan"), dtype=torch.float32, device="cuda")
    paged = None
    kc, vc = dev["k_cache"].data_ptr(), dev["v_cache"].data_ptr()
    if page_size is not None:
        kp, vp, table, num_pages = _paged(inp, page_size)

        def bf(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)

        kp_d, vp_d = bf(kp), bf(vp)
        tab_d = torch.from_numpy(table).cuda()
        paged = binding.PagedKV(page_size, table.shape[1], num_pages, tab_d.data_ptr())
        kc, vc = kp_d.data_ptr(), vp_d.data_ptr()
    stream = torch.cuda.current_stream().cuda_stream
    rc = binding.call_ex_raw(dev["q"].data_ptr(), kc, vc, paged, dev["k_tree"].data_ptr(), dev["v_tree"].data_ptr(),
                             dev["parent"].data_ptr(), dev["cu_seqlens"].data_ptr(), tree, out.data_ptr(),
                             lse.data_ptr(), dims, ws.data_ptr(), wsb, stream)
    assert rc == expect_rc, binding.STATUS_NAMES.get(rc, rc)
    torch.cuda.synchronize()
    status = binding.check(dims, ws.data_ptr(), stream)
    o = out.float().cpu().numpy().astype(np.float64).reshape(-1, w.head_dim)
    l_ = lse.cpu().numpy().astype(np.float64).reshape(-1)
    q_after = dev["q"].view(torch.int16).cpu().numpy().view(np.uint16)
    return o, l_, status, q_after


def _oracle(inp, theta=0.0, window=0):
    w = inp.workload
    q, kt = inp.q, inp.k_tree
    if theta > 0:
        pos = tp.tree_positions(inp.parent, inp.cu_seqlens, inp.node_offsets())
        q, kt = tp.rope_bf16(q, pos, theta), tp.rope_bf16(kt, pos, theta)
    if window > 0:
        return oracle.verify_attn_oracle_window(q, inp.k_cache, inp.v_cache, kt, inp.v_tree, inp.parent,
                                                inp.cu_seqlens, inp.node_offsets(), num_q_heads=w.num_q_heads,
                                                num_kv_heads=w.num_kv_heads, head_dim=w.head_dim, scale=inp.scale,
                                                window=window)
    return oracle.verify_attn_oracle_packed(q, inp.k_cache, inp.v_cache, kt, inp.v_tree, inp.parent,
                                            inp.cu_seqlens, inp.node_offsets(), num_q_heads=w.num_q_heads,
                                            num_kv_heads=w.num_kv_heads, head_dim=w.head_dim, scale=inp.scale)


def _assert_close(o, l_, ro, rl):
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(l_))
    assert np.all(np.abs(o - ro) <= out_tolerance(ro))
    assert np.abs(l_ - rl).max() <= LSE_ATOL


@pytest.mark.parametrize("theta", [0.0, 1e6])
def test_ragged_trees_g7(theta):
    # g = 7: units of 36 nodes; trees of 1, 128 (four units), 37 (one past a unit), 0 and 72
    w = Workload("ragged_g7", 5, 28, 4, 128, 128, 0, "uniform", lengths=[3000, 0, 1000, 129, 5000],
                 tree_sizes=[1, 128, 37, 0, 72])
    inp = make_inputs(w, seed=21)
    o, l_, st, q_after = _run_ex(inp, theta)
    assert st == binding.LS_OK
    assert np.array_equal(q_after, inp.q)  # the rotation goes to the workspace, not into q
    ro, rl = _oracle(inp, theta)
    _assert_close(o, l_, ro, rl)


@pytest.mark.parametrize("theta", [0.0, 10000.0])
def test_ragged_trees_d64_device_lengths(theta):
    w = Workload("ragged_d64", 4, 8, 1, 64, 64, (0, 3000), "window8", tree_sizes=[33, 32, 64, 5])
    inp = make_inputs(w, seed=22)
    o, l_, st, _ = _run_ex(inp, theta, host_lengths=False)
    assert st == binding.LS_OK
    ro, rl = _oracle(inp, theta)
    _assert_close(o, l_, ro, rl)


@pytest.mark.parametrize("theta", [10000.0, 500000.0])
def test_rope_uniform_trees(theta):
    w = Workload("rope_llama", 2, 32, 8, 128, 64, 2000, "window8")
    inp = make_inputs(w, seed=23)
    o, l_, st, _ = _run_ex(inp, theta)
    assert st == binding.LS_OK
    ro, rl = _oracle(inp, theta)
    _assert_close(o, l_, ro, rl)


def test_rope_paged_ragged():
    w = Workload("rope_paged", 3, 16, 4, 128, 96, 0, "bfs", lengths=[700, 1, 2100], tree_sizes=[96, 40, 3])
    inp = make_inputs(w, seed=24)
    o, l_, st, _ = _run_ex(inp, 500000.0, page_size=16)
    assert st == binding.LS_OK
    ro, rl = _oracle(inp, 500000.0)
    _assert_close(o, l_, ro, rl)


def test_rope_long_prefix_all_rows():
    # positions near 64k: the angle reduction must keep its precision there
    w = Workload("rope_qwen", 1, 28, 4, 128, 64, 65536, "window8")
    inp = make_inputs(w, seed=25)
    theta = 1e6
    o, l_, st, _ = _run_ex(inp, theta)
    assert st == binding.LS_OK
    pos = tp.tree_positions(inp.parent, inp.cu_seqlens, inp.node_offsets())
    qr, kr = tp.rope_bf16(inp.q, pos, theta), tp.rope_bf16(inp.k_tree, pos, theta)
    ro, rl = oracle.verify_attn_oracle(qr, inp.k_cache, inp.v_cache, kr, inp.v_tree, inp.parent, inp.cu_seqlens,
                                       num_q_heads=28, num_kv_heads=4, head_dim=128, tree_size=64)
    assert np.all(np.abs(o - ro) <= out_tolerance(ro))
    assert np.abs(l_ - rl).max() <= LSE_ATOL


def test_rope_bad_tree_reported():
    w = Workload("rope_bad", 2, 8, 2, 64, 8, 100, "chain")
    inp = make_inputs(w, seed=26)
    inp.parent[8 + 3] = 5  # node 3 of sequence 1 points below itself
    _, _, st, _ = _run_ex(inp, 10000.0)
    assert st == 5  # LS_ERR_BAD_TREE


def test_bad_device_cu_tree_reported():
    w = Workload("bad_cu_tree", 2, 8, 2, 64, 16, 300, "chain", tree_sizes=[5, 9])
    inp = make_inputs(w, seed=27)
    bad = torch.tensor([0, 9, 5], dtype=torch.int32, device="cuda")  # decreasing: not a packed layout
    _, _, st, _ = _run_ex(inp, 0.0, cu_tree_dev=bad)
    assert st == 7  # LS_ERR_LENGTHS
    _, _, st, _ = _run_ex(inp, 10000.0, cu_tree_dev=torch.tensor([0, 5, 15], dtype=torch.int32, device="cuda"))
    assert st == 7  # cu_tree[B] differs from total_nodes


def test_host_checks_of_tree_options():
    dims, keep = binding.make_dims(2, 8, 2, 64, 16, max_prefix_len=100)
    cu = torch.tensor([0, 5, 9], dtype=torch.int32, device="cuda")
    too_many = binding.TreeOpts(cu_tree=cu.data_ptr(), total_nodes=33)  # more than B * T nodes
    assert binding.ex_workspace_size(dims, too_many) == 0
    assert binding.ex_workspace_size(dims, binding.TreeOpts(rope_theta=0.5)) == 0  # base <= 1
    assert binding.ex_workspace_size(dims, binding.TreeOpts(rope_theta=float("nan"))) == 0
    plain = binding.ex_workspace_size(dims, None)
    assert plain == binding.workspace_size(dims)
    assert binding.ex_workspace_size(dims, binding.TreeOpts(rope_theta=10000.0)) > plain
    assert binding.ex_workspace_size(dims, binding.TreeOpts(window=15)) == 0  # shorter than the tree
    assert binding.ex_workspace_size(dims, binding.TreeOpts(window=-1)) == 0
    assert 0 < binding.ex_workspace_size(dims, binding.TreeOpts(window=16)) <= plain


# ----------------------------------------------------------------------------- sliding window
@pytest.mark.parametrize("window,lengths", [
    (512, [3000, 700, 0, 511]),   # full windows, one just short, no prefix, L = W - 1
    (129, [1000, 5, 260, 129]),   # per-row cuts up to 231 keys: across two key blocks
    (64, [64, 63, 65, 192]),      # the smallest window for 64 nodes
])
def test_sliding_window(window, lengths):
    w = Workload("win", 4, 8, 2, 128, 64, 0, "window8", lengths=lengths)
    inp = make_inputs(w, seed=31)
    o, l_, st, _ = _run_ex(inp, window=window)
    assert st == binding.LS_OK
    ro, rl = _oracle(inp, window=window)
    _assert_close(o, l_, ro, rl)


@pytest.mark.parametrize("page_size", [16, 256])
def test_sliding_window_paged_ragged_rope(page_size):
    w = Workload("win_paged", 3, 28, 4, 128, 128, 0, "bfs", lengths=[4100, 300, 777], tree_sizes=[128, 37, 1])
    inp = make_inputs(w, seed=32)
    o, l_, st, _ = _run_ex(inp, 500000.0, page_size=page_size, window=300)
    assert st == binding.LS_OK
    ro, rl = _oracle(inp, 500000.0, window=300)
    _assert_close(o, l_, ro, rl)


def test_sliding_window_d64_device_lengths():
    w = Workload("win64", 2, 4, 1, 64, 16, 0, "uniform", lengths=[2000, 200])
    inp = make_inputs(w, seed=33)
    o, l_, st, _ = _run_ex(inp, window=100, host_lengths=False)
    assert st == binding.LS_OK
    ro, rl = _oracle(inp, window=100)
    _assert_close(o, l_, ro, rl)


@pytest.mark.parametrize("B,Hq,Hkv,d,T,lengths", [(2, 28, 4, 128, 64, [3000, 9000]),
                                                   (3, 8, 2, 64, 16, [130, 0, 5000]),
                                                   (2, 28, 4, 128, 64, [3072, 8960])])
def test_plain_and_general_instances_agree_bitwise(B, Hq, Hkv, d, T, lengths):
    """The partials kernel is compiled twice: a plain instance (packed cache, whole prefix,
    inputs as given) and a general one (paged caches, windows, rotation). A window longer
    than every key list asks for the general instance without changing what is computed,
    or where the keys sit in a block: it must give the plain call's bits. So must a paged
    cache of 128-key pages when every length is a multiple of 128 (otherwise its last
    block holds the keys at other columns, masked at the end instead of the start, and
    the sums round differently)."""
    w = Workload("instances", B, Hq, Hkv, d, T, 0, "window8", input_scale=1.0, lengths=lengths)
    inp = make_inputs(w, seed=30 + d)
    o_plain, l_plain, st, _ = _run_ex(inp)
    assert st == binding.LS_OK
    o_win, l_win, st, _ = _run_ex(inp, window=max(lengths) + T + 1)
    assert st == binding.LS_OK
    np.testing.assert_array_equal(o_win, o_plain)
    np.testing.assert_array_equal(l_win, l_plain)
    o_pg, l_pg, st, _ = _run_ex(inp, page_size=128)
    assert st == binding.LS_OK
    if all(L % 128 == 0 for L in lengths):
        np.testing.assert_array_equal(o_pg, o_plain)
        np.testing.assert_array_equal(l_pg, l_plain)
    ro, rl = _oracle(inp)
    _assert_close(o_plain, l_plain, ro, rl)
    _assert_close(o_pg, l_pg, ro, rl)
