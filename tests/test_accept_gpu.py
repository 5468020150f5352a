"""GPU parity of greedy tree acceptance (ls_tree_accept_greedy) against the oracle
(oracle/accept.py): accepted count, path and next token must match exactly (integer
results; the argmax compares the logits in their own dtype on both sides)."""
from __future__ import annotations

import json
import os

import numpy as np
import pytest
import torch

from oracle import accept as oa
from tree_verification_attention_longspec_b200 import binding
from tree_verification_attention_longspec_b200.inputs import AcceptInputs, bf16_bits_from_f32, make_accept_inputs

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_accept.json")


def _run(inp, misalign=False):
    """Returns [(len, path, next)] per sequence from the GPU."""
    if inp.dtype == "bf16":
        host = torch.from_numpy(np.ascontiguousarray(inp.logits).view(np.int16))
        elem, dt = 2, binding.LS_DTYPE_BF16
    else:
        host = torch.from_numpy(np.ascontiguousarray(inp.logits, dtype=np.float32))
        elem, dt = 4, binding.LS_DTYPE_F32
    N, V = inp.logits.shape
    if misalign:  # rows off 16-byte boundaries: the kernel must take the scalar path
        buf = torch.zeros(N * V + 1, dtype=host.dtype, device="cuda")
        buf[1:].copy_(host.reshape(-1).cuda())
        lptr = buf.data_ptr() + elem
    else:
        buf = host.cuda()
        lptr = buf.data_ptr()
    tok = torch.from_numpy(inp.tokens.astype(np.int32)).cuda()
    par = torch.from_numpy(inp.parent.astype(np.int32)).cuda()
    cu = torch.from_numpy(inp.cu_tree.astype(np.int32)).cuda() if inp.cu_tree is not None else None
    dims = binding.AcceptDims(inp.batch, inp.tree_size, inp.vocab, dt)
    wsb = binding.accept_workspace_size(dims, N)
    assert wsb > 0
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    alen = torch.full((inp.batch,), -7, dtype=torch.int32, device="cuda")
    path = torch.full((inp.batch, inp.tree_size), -7, dtype=torch.int32, device="cuda")
    nxt = torch.full((inp.batch,), -7, dtype=torch.int32, device="cuda")
    rc = binding.call_accept_raw(lptr, tok.data_ptr(), par.data_ptr(), cu.data_ptr() if cu is not None else None,
                                 N, alen.data_ptr(), path.data_ptr(), nxt.data_ptr(), dims, ws.data_ptr(), wsb,
                                 torch.cuda.current_stream().cuda_stream)
    assert rc == binding.LS_OK
    torch.cuda.synchronize()
    a, p, x = alen.cpu().numpy(), path.cpu().numpy(), nxt.cpu().numpy()
    out = []
    for b in range(inp.batch):
        n = int(a[b])
        out.append((n, [int(v) for v in p[b, : n + 1]] if n >= 0 else [], int(x[b])))
    return out


def _check(inp, **kw):
    got = _run(inp, **kw)
    want = oa.accept_greedy(inp)
    assert got == [(n, list(pth), int(nx)) for n, pth, nx in want]
    return got


def test_hand_worked_example():
    with open(GOLDEN) as f:
        g = json.load(f)
    logits = np.array([[float(x) for x in row] for row in g["logits"]], dtype=np.float32)
    inp = AcceptInputs(logits, np.array(g["tokens"], np.int32), np.array(g["parent"], np.int32),
                       np.array(g["cu_tree"], np.int32), len(g["cu_tree"]) - 1, g["tree_size"], g["vocab"], "f32")
    got = _check(inp)
    assert [r[0] for r in got] == [e["accept_len"] for e in g["expected"]]
    inp.logits, inp.dtype = bf16_bits_from_f32(logits), "bf16"
    _check(inp)


def test_qwen_vocab_bf16():
    inp = make_accept_inputs(1, 64, 152064, "bf16", match_prob=0.8, seed=0)
    got = _check(inp)
    assert got[0][0] >= 1


def test_llama_vocab_fp32_ragged():
    inp = make_accept_inputs(4, 128, 128256, "f32", tree="bfs", match_prob=0.9, seed=1,
                             tree_sizes=[128, 1, 0, 77])
    got = _check(inp)
    assert got[1][0] == 0 and got[2][0] == -1


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_odd_vocab_and_misaligned_rows(dtype):
    inp = make_accept_inputs(3, 16, 32003, dtype, tree="uniform", match_prob=0.8, seed=2)
    _check(inp)
    inp = make_accept_inputs(2, 16, 32000, dtype, tree="uniform", match_prob=0.8, seed=3)
    _check(inp, misalign=True)


def test_ties_across_segments():
    # every row holds its maximum twice, far apart (different segments of the row): the
    # first index must win
    inp = make_accept_inputs(2, 32, 152064, "f32", tree="window8", match_prob=0.0, seed=4)
    rng = np.random.default_rng(4)
    for r in range(inp.logits.shape[0]):
        i, j = sorted(rng.choice(152064, size=2, replace=False))
        inp.logits[r, i] = inp.logits[r, j] = 9.0
        kids = np.nonzero(inp.parent[(r // 32) * 32:(r // 32 + 1) * 32] == r % 32)[0]
        for k in kids:  # children carry one of the two tied tokens
            inp.tokens[(r // 32) * 32 + k] = i if rng.random() < 0.5 else j
    _check(inp)


def test_nan_and_inf_rows():
    inp = make_accept_inputs(1, 8, 4096, "f32", tree="chain", match_prob=1.0, seed=5)
    inp.logits[0, :] = -np.inf
    inp.tokens[1] = 0          # all -inf: argmax 0, node 1 accepted
    inp.logits[1, ::2] = np.nan
    _check(inp)


def test_bad_tree():
    inp = make_accept_inputs(2, 8, 1000, "bf16", tree="chain", seed=6)
    inp.parent[8 + 3] = 3
    got = _check(inp)
    assert got[1] == (-1, [], -1) and got[0][0] >= 0
