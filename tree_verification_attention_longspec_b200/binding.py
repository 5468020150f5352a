"""Thin Python binding of the C-ABI library (argument marshalling only).

Every step of the computation runs in the CUDA kernels of ``libls_verify_attn.so``;
this module checks torch tensors, takes their device pointers and the current
stream, and calls the C functions declared in ``include/ls_verify_attn.h``. There is
no fallback: if the library is missing or the call fails, it raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libls_verify_attn.so")
# the index-checking build of the same sources (tests only): see build.py --debug
DEBUG_LIB_PATH = os.path.join(_HERE, "lib", "libls_verify_attn_debug.so")

LS_OK = 0
STATUS_NAMES = {0: "LS_OK", 1: "LS_ERR_INVALID_ARG", 2: "LS_ERR_UNSUPPORTED", 3: "LS_ERR_WORKSPACE",
                4: "LS_ERR_CUDA", 5: "LS_ERR_BAD_TREE", 6: "LS_ERR_TIMEOUT", 7: "LS_ERR_LENGTHS",
                8: "LS_ERR_INDEX"}
EXPORTED = ("ls_verify_attn", "ls_verify_attn_partials", "ls_verify_attn_combine",
            "ls_verify_attn_workspace_size", "ls_verify_attn_check", "ls_status_string",
            "ls_verify_attn_plan", "ls_verify_attn_static", "ls_verify_attn_paged", "ls_cross_attn",
            "ls_cross_attn_workspace_size", "ls_verify_attn_ex", "ls_verify_attn_ex_workspace_size",
            "ls_tree_accept_greedy", "ls_tree_accept_workspace_size")
LS_DTYPE_BF16, LS_DTYPE_F32 = 0, 1


class LSError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        name = STATUS_NAMES.get(status, str(status))
        msg = f"{name}"
        try:
            msg += f" ({load_library().ls_status_string(status).decode()})"
        except Exception:
            pass
        super().__init__(f"{what}: {msg}" if what else msg)


class PagedKV(ctypes.Structure):
    _fields_ = [("page_size", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
                ("num_pages", ctypes.c_int64), ("page_table", ctypes.c_void_p)]


class TreeOpts(ctypes.Structure):
    """ls_tree_opts: per-sequence trees (cu_tree, device address), sliding window, in-kernel RoPE,
    and the limit of the kernel's device-side waits (0: the default, 4 s)."""
    _fields_ = [("cu_tree", ctypes.c_void_p), ("total_nodes", ctypes.c_int32), ("window", ctypes.c_int32),
                ("rope_theta", ctypes.c_double), ("wait_limit_ns", ctypes.c_uint64)]


class AcceptDims(ctypes.Structure):
    """ls_accept_dims of the greedy acceptance call."""
    _fields_ = [("batch", ctypes.c_int32), ("tree_size", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("logits_dtype", ctypes.c_int32)]


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("tree_size", ctypes.c_int32), ("max_prefix_len", ctypes.c_int32),
                ("cu_seqlens_host", ctypes.POINTER(ctypes.c_int32)),
                ("softmax_scale", ctypes.c_float)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load the CUDA library. Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    _lib = _open(path)
    return _lib


def load_debug_library(path: str = DEBUG_LIB_PATH):
    """Load the index-checking build (a separate library with the same entry points,
    not the one the other calls here use). Raises if it has not been built."""
    return _open(path)


def _open(path: str):
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m tree_verification_attention_longspec_b200.build`")
    lib = ctypes.CDLL(path)
    P, D = ctypes.c_void_p, ctypes.POINTER(Dims)
    lib.ls_verify_attn.argtypes = [P, P, P, P, P, P, P, P, P, D, P, ctypes.c_size_t, P]
    lib.ls_verify_attn.restype = ctypes.c_int
    lib.ls_verify_attn_partials.argtypes = [P, P, P, P, P, P, P, D, P, ctypes.c_size_t, P]
    lib.ls_verify_attn_partials.restype = ctypes.c_int
    lib.ls_verify_attn_combine.argtypes = [P, P, P, D, P, ctypes.c_size_t, P]
    lib.ls_verify_attn_combine.restype = ctypes.c_int
    lib.ls_verify_attn_paged.argtypes = [P, P, P, ctypes.POINTER(PagedKV), P, P, P, P, P, P, D, P,
                                         ctypes.c_size_t, P]
    lib.ls_verify_attn_paged.restype = ctypes.c_int
    lib.ls_cross_attn.argtypes = [P, P, P, P, P, P, D, P, ctypes.c_size_t, P]
    lib.ls_cross_attn.restype = ctypes.c_int
    lib.ls_cross_attn_workspace_size.argtypes = [D]
    lib.ls_cross_attn_workspace_size.restype = ctypes.c_size_t
    T = ctypes.POINTER(TreeOpts)
    lib.ls_verify_attn_ex.argtypes = [P, P, P, ctypes.POINTER(PagedKV), P, P, P, P, T, P, P, D, P,
                                      ctypes.c_size_t, P]
    lib.ls_verify_attn_ex.restype = ctypes.c_int
    lib.ls_verify_attn_ex_workspace_size.argtypes = [D, T]
    lib.ls_verify_attn_ex_workspace_size.restype = ctypes.c_size_t
    A = ctypes.POINTER(AcceptDims)
    lib.ls_tree_accept_workspace_size.argtypes = [A, ctypes.c_int32]
    lib.ls_tree_accept_workspace_size.restype = ctypes.c_size_t
    lib.ls_tree_accept_greedy.argtypes = [P, P, P, P, ctypes.c_int32, P, P, P, A, P, ctypes.c_size_t, P]
    lib.ls_tree_accept_greedy.restype = ctypes.c_int
    lib.ls_verify_attn_static.argtypes = [P, P, P, P, P, P, P, P, P, D, P]
    lib.ls_verify_attn_static.restype = ctypes.c_int
    lib.ls_verify_attn_workspace_size.argtypes = [D]
    lib.ls_verify_attn_workspace_size.restype = ctypes.c_size_t
    lib.ls_verify_attn_check.argtypes = [D, P, P]
    lib.ls_verify_attn_check.restype = ctypes.c_int
    lib.ls_status_string.argtypes = [ctypes.c_int]
    lib.ls_status_string.restype = ctypes.c_char_p
    I = ctypes.POINTER(ctypes.c_int32)
    lib.ls_verify_attn_plan.argtypes = [D, I, I, I]
    lib.ls_verify_attn_plan.restype = ctypes.c_int
    return lib


def make_dims(batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int, tree_size: int,
              max_prefix_len: int = 0, cu_seqlens_host: Optional[Sequence[int]] = None,
              softmax_scale: float = 0.0):
    """Build the C dims struct. Returns (dims, keepalive) — keep both alive while used."""
    keep = None
    ptr = None
    if cu_seqlens_host is not None:
        keep = np.ascontiguousarray(np.asarray(cu_seqlens_host), dtype=np.int32)
        ptr = keep.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
        if max_prefix_len == 0 and len(keep) > 1:
            max_prefix_len = int(np.max(np.diff(keep)))
    d = Dims(batch, num_q_heads, num_kv_heads, head_dim, tree_size, max_prefix_len, ptr,
             float(softmax_scale))
    return d, keep


def workspace_size(dims: Dims) -> int:
    return int(load_library().ls_verify_attn_workspace_size(ctypes.byref(dims)))


def plan(dims: Dims):
    a, b, c = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    rc = load_library().ls_verify_attn_plan(ctypes.byref(dims), ctypes.byref(a), ctypes.byref(b),
                                            ctypes.byref(c))
    if rc != LS_OK:
        raise LSError(rc, "ls_verify_attn_plan")
    return {"partials_ctas": a.value, "blocks_per_chunk": b.value, "combine_ctas": c.value}


def call_raw(q, k_cache, v_cache, k_tree, v_tree, parent, cu_seqlens, out, lse, dims: Dims,
             workspace, workspace_bytes: int, stream) -> int:
    """ls_verify_attn on raw device addresses (ints); returns the status code."""
    return int(load_library().ls_verify_attn(q, k_cache, v_cache, k_tree, v_tree, parent,
                                             cu_seqlens, out, lse, ctypes.byref(dims), workspace,
                                             workspace_bytes, stream))


def call_static_raw(q, k_cache, v_cache, k_tree, v_tree, parent, cu_seqlens, out, lse, dims: Dims,
                    stream) -> int:
    """ls_verify_attn_static on raw device addresses (ints): no workspace argument, for
    callers that cannot allocate device memory; returns the status code."""
    return int(load_library().ls_verify_attn_static(q, k_cache, v_cache, k_tree, v_tree, parent,
                                                    cu_seqlens, out, lse, ctypes.byref(dims), stream))


def call_paged_raw(q, k_pages, v_pages, paged: PagedKV, k_tree, v_tree, parent, cu_seqlens, out, lse,
                   dims: Dims, workspace, workspace_bytes: int, stream) -> int:
    """ls_verify_attn_paged on raw device addresses (ints); returns the status code."""
    return int(load_library().ls_verify_attn_paged(q, k_pages, v_pages, ctypes.byref(paged), k_tree, v_tree,
                                                   parent, cu_seqlens, out, lse, ctypes.byref(dims), workspace,
                                                   workspace_bytes, stream))


def ex_workspace_size(dims: Dims, tree: Optional[TreeOpts]) -> int:
    return int(load_library().ls_verify_attn_ex_workspace_size(ctypes.byref(dims),
                                                               None if tree is None else ctypes.byref(tree)))


def call_ex_raw(q, k_cache, v_cache, paged: Optional[PagedKV], k_tree, v_tree, parent, cu_seqlens,
                tree: Optional[TreeOpts], out, lse, dims: Dims, workspace, workspace_bytes: int, stream) -> int:
    """ls_verify_attn_ex (paged cache, per-sequence trees, in-kernel RoPE) on raw device addresses."""
    return int(load_library().ls_verify_attn_ex(q, k_cache, v_cache, None if paged is None else ctypes.byref(paged),
                                                k_tree, v_tree, parent, cu_seqlens,
                                                None if tree is None else ctypes.byref(tree), out, lse,
                                                ctypes.byref(dims), workspace, workspace_bytes, stream))


def accept_workspace_size(dims: AcceptDims, total_nodes: int) -> int:
    return int(load_library().ls_tree_accept_workspace_size(ctypes.byref(dims), int(total_nodes)))


def call_accept_raw(logits, tokens, parent, cu_tree, total_nodes: int, accept_len, accept_path, next_token,
                    dims: AcceptDims, workspace, workspace_bytes: int, stream) -> int:
    """ls_tree_accept_greedy on raw device addresses; returns the status code."""
    return int(load_library().ls_tree_accept_greedy(logits, tokens, parent, cu_tree, int(total_nodes), accept_len,
                                                    accept_path, next_token, ctypes.byref(dims), workspace,
                                                    workspace_bytes, stream))


def cross_workspace_size(dims: Dims) -> int:
    return int(load_library().ls_cross_attn_workspace_size(ctypes.byref(dims)))


def call_cross_raw(q, k_cache, v_cache, cu_seqlens, out, lse, dims: Dims, workspace, workspace_bytes: int,
                   stream) -> int:
    """ls_cross_attn (prefix-only attention) on raw device addresses; returns the status code."""
    return int(load_library().ls_cross_attn(q, k_cache, v_cache, cu_seqlens, out, lse, ctypes.byref(dims),
                                            workspace, workspace_bytes, stream))


def call_partials_raw(q, k_cache, v_cache, k_tree, v_tree, parent, cu_seqlens, dims: Dims, workspace,
                      workspace_bytes: int, stream) -> int:
    """ls_verify_attn_partials (the dominant kernel) on raw device addresses."""
    return int(load_library().ls_verify_attn_partials(q, k_cache, v_cache, k_tree, v_tree, parent,
                                                      cu_seqlens, ctypes.byref(dims), workspace,
                                                      workspace_bytes, stream))


def call_combine_raw(cu_seqlens, out, lse, dims: Dims, workspace, workspace_bytes: int, stream) -> int:
    """ls_verify_attn_combine on raw device addresses."""
    return int(load_library().ls_verify_attn_combine(cu_seqlens, out, lse, ctypes.byref(dims), workspace,
                                                     workspace_bytes, stream))


def check(dims: Dims, workspace_ptr: int, stream_ptr: int) -> int:
    return int(load_library().ls_verify_attn_check(ctypes.byref(dims), workspace_ptr, stream_ptr))


def _dev_ptr(t, name, dtype, nbytes_elem):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


class VerifyAttn:
    """A reusable call: fixed dims, one workspace, any inputs of those shapes."""

    def __init__(self, batch, num_q_heads, num_kv_heads, head_dim, tree_size, *,
                 cu_seqlens_host=None, max_prefix_len=0, softmax_scale=0.0, device=None):
        import torch
        self.dims, self._keep = make_dims(batch, num_q_heads, num_kv_heads, head_dim, tree_size,
                                          max_prefix_len, cu_seqlens_host, softmax_scale)
        self.ws_bytes = workspace_size(self.dims)
        if self.ws_bytes == 0:
            raise LSError(1, "ls_verify_attn_workspace_size returned 0 (invalid or unsupported dims)")
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8,
                                     device=device if device is not None else "cuda")
        self.plan = plan(self.dims)

    def __call__(self, q, k_cache, v_cache, k_tree, v_tree, parent, cu_seqlens, out=None, lse=None,
                 stream=None):
        import torch
        bf = torch.bfloat16
        d = self.dims
        if out is None:
            out = torch.empty_like(q)
        if lse is None:
            lse = torch.empty(q.shape[0], d.num_q_heads, dtype=torch.float32, device=q.device)
        ptrs = [_dev_ptr(q, "q", bf, 2), _dev_ptr(k_cache, "k_cache", bf, 2),
                _dev_ptr(v_cache, "v_cache", bf, 2), _dev_ptr(k_tree, "k_tree", bf, 2),
                _dev_ptr(v_tree, "v_tree", bf, 2), _dev_ptr(parent, "tree_parent", torch.int32, 4),
                _dev_ptr(cu_seqlens, "cu_seqlens", torch.int32, 4), _dev_ptr(out, "out", bf, 2),
                _dev_ptr(lse, "lse", torch.float32, 4)]
        if stream is None:
            stream = torch.cuda.current_stream(q.device)
        sp = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        rc = call_raw(*ptrs, d, self.workspace.data_ptr(), self.ws_bytes, sp)
        if rc != LS_OK:
            raise LSError(rc, "ls_verify_attn")
        return out, lse

    def check(self, stream=None) -> int:
        import torch
        if stream is None:
            stream = torch.cuda.current_stream(self.workspace.device)
        sp = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        return check(self.dims, self.workspace.data_ptr(), sp)


def verify_attn(q, k_cache, v_cache, k_tree, v_tree, tree_parent, cu_seqlens, *, tree_size: int,
                num_kv_heads: int, cu_seqlens_host=None, max_prefix_len: int = 0,
                softmax_scale: float = 0.0, out=None, lse=None, check_status: bool = False):
    """One call of tree-verification attention on torch CUDA tensors.

    q [B*T, H_q, d] bf16; k_cache/v_cache [sum L_b, H_kv, d] bf16; k_tree/v_tree
    [B*T, H_kv, d] bf16; tree_parent [B*T] int32; cu_seqlens [B+1] int32 (device).
    Returns (out [B*T, H_q, d] bf16, lse [B*T, H_q] fp32).
    """
    B = int(cu_seqlens.shape[0]) - 1
    op = VerifyAttn(B, int(q.shape[1]), num_kv_heads, int(q.shape[2]), tree_size,
                    cu_seqlens_host=cu_seqlens_host, max_prefix_len=max_prefix_len,
                    softmax_scale=softmax_scale, device=q.device)
    out, lse = op(q, k_cache, v_cache, k_tree, v_tree, tree_parent, cu_seqlens, out, lse)
    if check_status:
        rc = op.check()
        if rc != LS_OK:
            raise LSError(rc, "device status")
    return out, lse
