"""Python binding of libtlsp (include/tlsp.h): argument marshalling only.

Every step of the path runs in the CUDA library; this module only turns
torch tensors into device pointers, allocates outputs and the workspace with
PyTorch, and passes the current CUDA stream. It fails loudly when the library
is missing: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtlsp.so")

TLSP_OK = 0
TLSP_ERR_INVALID_ARG = -1
TLSP_ERR_UNSUPPORTED = -2
TLSP_ERR_WORKSPACE = -3
TLSP_ERR_CUDA = -4
TLSP_ERR_TIMEOUT = -5
TLSP_ERR_DEVICE_ASSERT = -6

TLSP_F32 = 0
TLSP_BF16 = 1

EXPORTED = [
    "tlsp_num_groups", "tlsp_num_levels", "tlsp_workspace_bytes", "tlsp_group_queries",
    "tlsp_group_queries_trace", "tlsp_split_from_projections", "tlsp_anchor_attention",
    "tlsp_reuse_attention", "tlsp_dense_attention", "tlsp_dense_attention_noalloc",
    "tlsp_topk_from_scores", "tlsp_get_device_status",
    "tlsp_reset_device_status", "tlsp_debug_bounded_wait", "tlsp_status_string",
    "tlsp_last_cuda_error", "tlsp_launch_count", "tlsp_group_raster",
    "tlsp_block_topk_from_scores", "tlsp_pooled_block_select",
]


class TlspError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})")


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("n_q", ctypes.c_int32),
                ("n_kv", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("dtype", ctypes.c_int)]


_lib = None


def lib() -> ctypes.CDLL:
    """Loads the in-tree libtlsp.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m token_level_sparse_pddp_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        dp = ctypes.POINTER(Dims)
        sig = {
            "tlsp_num_groups": (i32, [i32, i32]),
            "tlsp_num_levels": (i32, [i32, i32]),
            "tlsp_workspace_bytes": (sz, [dp, i32, i32]),
            "tlsp_group_queries": (ctypes.c_int, [dp, vp, i32, vp, vp, sz, vp]),
            "tlsp_group_queries_trace": (ctypes.c_int, [dp, vp, i32, vp, vp, vp, sz, vp]),
            "tlsp_split_from_projections": (ctypes.c_int, [vp, vp, i32, i32, vp, vp, vp, sz, vp]),
            "tlsp_anchor_attention": (ctypes.c_int,
                                      [dp, vp, vp, vp, vp, i32, i32, vp, vp, vp, vp, vp, sz, vp]),
            "tlsp_reuse_attention": (ctypes.c_int,
                                     [dp, vp, vp, vp, vp, i32, i32, vp, vp, vp, vp, sz, vp]),
            "tlsp_dense_attention": (ctypes.c_int, [dp, vp, vp, vp, vp, vp, vp, sz, vp]),
            "tlsp_dense_attention_noalloc": (ctypes.c_int, [dp, vp, vp, vp, vp, vp]),
            "tlsp_topk_from_scores": (ctypes.c_int, [vp, i32, i32, i32, vp, vp, sz, vp]),
            "tlsp_get_device_status": (ctypes.c_int, [vp]),
            "tlsp_reset_device_status": (ctypes.c_int, [vp, vp]),
            "tlsp_debug_bounded_wait": (ctypes.c_int, [vp, sz, i64, vp]),
            "tlsp_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "tlsp_last_cuda_error": (ctypes.c_int, []),
            "tlsp_launch_count": (i64, []),
            "tlsp_group_raster": (ctypes.c_int, [dp, i32, vp, vp]),
            "tlsp_block_topk_from_scores": (ctypes.c_int, [vp, i32, i32, i32, i32, vp, vp, vp]),
            "tlsp_pooled_block_select": (ctypes.c_int,
                                         [dp, vp, vp, vp, i32, i32, i32, vp, vp, vp, sz, vp]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().tlsp_status_string(code).decode()


def _check(code: int, what: str):
    if code != TLSP_OK:
        if code == TLSP_ERR_CUDA:
            what += f" (cudaError {lib().tlsp_last_cuda_error()})"
        raise TlspError(code, what)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on the CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return TLSP_F32
    if dt == torch.bfloat16:
        return TLSP_BF16
    raise ValueError(f"unsupported dtype {dt}")


def dims_of(Q: torch.Tensor, K: Optional[torch.Tensor] = None) -> Dims:
    B, H, n_q, d = Q.shape
    n_kv = K.shape[2] if K is not None else n_q
    return Dims(B, H, n_q, n_kv, d, _dtype_code(Q.dtype))


def num_groups(n_q: int, group_size: int) -> int:
    return lib().tlsp_num_groups(n_q, group_size)


def num_levels(n_q: int, group_size: int) -> int:
    return lib().tlsp_num_levels(n_q, group_size)


def launch_count() -> int:
    return lib().tlsp_launch_count()


class Workspace:
    """Caller-owned scratch for the library calls (a zeroed torch byte tensor)."""

    def __init__(self, dims: Optional[Dims], group_size: int = 1, k: int = 1, device=None,
                 nbytes: Optional[int] = None):
        n = nbytes if nbytes is not None else lib().tlsp_workspace_bytes(
            ctypes.byref(dims), group_size, k)
        if n == 0:
            raise TlspError(TLSP_ERR_INVALID_ARG, "tlsp_workspace_bytes")
        self.nbytes = n
        self.buf = torch.zeros(n, dtype=torch.uint8, device=device or "cuda")

    @classmethod
    def status_only(cls, device=None) -> "Workspace":
        """The 256-byte workspace that the reuse step needs (its status word only)."""
        return cls(None, nbytes=256, device=device)

    @property
    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())

    def status(self) -> int:
        return lib().tlsp_get_device_status(self.ptr)

    def reset(self):
        _check(lib().tlsp_reset_device_status(self.ptr, _stream()), "tlsp_reset_device_status")


def group_queries(Q: torch.Tensor, group_size: int, ws: Workspace, trace: bool = False,
                  out: Optional[torch.Tensor] = None):
    """PDDP grouping -> groups int32 [B, H, G*group_size] (and per-level projections)."""
    d = dims_of(Q)
    G = num_groups(d.n_q, group_size)
    groups = (torch.empty((d.batch, d.heads, G * group_size), dtype=torch.int32, device=Q.device)
              if out is None else out)
    if trace:
        L = num_levels(d.n_q, group_size)
        proj = torch.empty((max(L, 0), d.batch, d.heads, d.n_q), dtype=torch.float32,
                           device=Q.device)
        _check(lib().tlsp_group_queries_trace(ctypes.byref(d), _ptr(Q), group_size, _ptr(groups),
                                              _ptr(proj) if L > 0 else ctypes.c_void_p(
                                                  groups.data_ptr()),
                                              ws.ptr, ws.nbytes, _stream()),
               "tlsp_group_queries_trace")
        return groups, proj
    _check(lib().tlsp_group_queries(ctypes.byref(d), _ptr(Q), group_size, _ptr(groups), ws.ptr,
                                    ws.nbytes, _stream()), "tlsp_group_queries")
    return groups


def anchor_attention(Q, K, V, groups, group_size: int, k: int, ws: Workspace,
                     return_scores: bool = False, out=None):
    """Anchor step -> (O_full, indices, R[, scores])."""
    d = dims_of(Q, K)
    G = num_groups(d.n_q, group_size)
    if out is None:
        O = torch.empty_like(Q)
        idx = torch.empty((d.batch, d.heads, G, k), dtype=torch.int32, device=Q.device)
        R = torch.empty(Q.shape, dtype=torch.float32, device=Q.device)
    else:
        O, idx, R = out
    S = (torch.empty((d.batch, d.heads, G, d.n_kv), dtype=torch.float32, device=Q.device)
         if return_scores else None)
    _check(lib().tlsp_anchor_attention(ctypes.byref(d), _ptr(Q), _ptr(K), _ptr(V), _ptr(groups),
                                       group_size, k, _ptr(O), _ptr(idx), _ptr(R), _ptr(S),
                                       ws.ptr, ws.nbytes, _stream()), "tlsp_anchor_attention")
    return (O, idx, R, S) if return_scores else (O, idx, R)


def reuse_attention(Q, K, V, groups, group_size: int, k: int, indices, R, ws: Workspace,
                    out: Optional[torch.Tensor] = None):
    """Reuse step -> O = sparse attention over the anchor's selection + R."""
    d = dims_of(Q, K)
    O = torch.empty_like(Q) if out is None else out
    _check(lib().tlsp_reuse_attention(ctypes.byref(d), _ptr(Q), _ptr(K), _ptr(V), _ptr(groups),
                                      group_size, k, _ptr(indices), _ptr(R), _ptr(O), ws.ptr,
                                      ws.nbytes, _stream()), "tlsp_reuse_attention")
    return O


def dense_attention(Q, K, V, ws: Workspace, out=None, lse=None):
    """Dense attention alone -> O (and fills lse [B, H, n_q] if given)."""
    d = dims_of(Q, K)
    O = torch.empty_like(Q) if out is None else out
    _check(lib().tlsp_dense_attention(ctypes.byref(d), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                      _ptr(lse), ws.ptr, ws.nbytes, _stream()),
           "tlsp_dense_attention")
    return O


def dense_attention_noalloc(Q, K, V, out=None):
    """Dense attention through the entry point that allocates nothing (fixed library scratch)."""
    d = dims_of(Q, K)
    O = torch.empty_like(Q) if out is None else out
    _check(lib().tlsp_dense_attention_noalloc(ctypes.byref(d), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                              _stream()), "tlsp_dense_attention_noalloc")
    return O


def topk_from_scores(scores: torch.Tensor, k: int, ws: Optional[Workspace] = None) -> torch.Tensor:
    """Per row of fp32 scores [..., n_kv]: ascending indices of the k largest (ties: lower index).

    With a workspace, a timed-out wait inside the kernel is recorded in its status word."""
    n_kv = scores.shape[-1]
    rows = scores.numel() // n_kv
    idx = torch.empty(scores.shape[:-1] + (k,), dtype=torch.int32, device=scores.device)
    wsp, wsn = (ws.ptr, ws.nbytes) if ws is not None else (None, 0)
    _check(lib().tlsp_topk_from_scores(_ptr(scores), rows, n_kv, k, _ptr(idx), wsp, wsn,
                                       _stream()),
           "tlsp_topk_from_scores")
    return idx


def split_from_projections(proj: torch.Tensor, members: torch.Tensor,
                           n_left: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """One PDDP cut of ascending `members` on proj[token] -> (left, right)."""
    n = members.numel()
    left = torch.empty(max(n_left, 1), dtype=torch.int32, device=members.device)
    right = torch.empty(max(n - n_left, 1), dtype=torch.int32, device=members.device)
    _check(lib().tlsp_split_from_projections(_ptr(proj), _ptr(members), n, n_left, _ptr(left),
                                             _ptr(right), None, 0, _stream()),
           "tlsp_split_from_projections")
    return left[:n_left], right[:n - n_left]


def debug_bounded_wait(ws: Workspace, spin_limit: int):
    _check(lib().tlsp_debug_bounded_wait(ws.ptr, ws.nbytes, spin_limit, _stream()),
           "tlsp_debug_bounded_wait")


# ----------------------------------------------------------------- ablation

def group_raster(Q: torch.Tensor, group_size: int, out: Optional[torch.Tensor] = None):
    """Raster query groups (consecutive tokens, no PDDP) -> int32 [B, H, G*group_size]."""
    d = dims_of(Q)
    G = num_groups(d.n_q, group_size)
    groups = (torch.empty((d.batch, d.heads, G * group_size), dtype=torch.int32, device=Q.device)
              if out is None else out)
    _check(lib().tlsp_group_raster(ctypes.byref(d), group_size, _ptr(groups), _stream()),
           "tlsp_group_raster")
    return groups


def block_topk_from_scores(scores: torch.Tensor, k: int, block: int,
                           return_block_scores: bool = False):
    """Block-granular selection from per-key scores [..., n_kv] -> indices [..., k]
    (and the block scores [..., n_kv / block] when asked)."""
    n_kv = scores.shape[-1]
    rows = scores.numel() // n_kv
    idx = torch.empty(scores.shape[:-1] + (k,), dtype=torch.int32, device=scores.device)
    bs = (torch.empty(scores.shape[:-1] + (n_kv // block,), dtype=torch.float32,
                      device=scores.device) if return_block_scores else None)
    _check(lib().tlsp_block_topk_from_scores(_ptr(scores), rows, n_kv, k, block, _ptr(idx),
                                             _ptr(bs), _stream()),
           "tlsp_block_topk_from_scores")
    return (idx, bs) if return_block_scores else idx


def pooled_block_select(Q: torch.Tensor, K: torch.Tensor, groups: torch.Tensor, group_size: int,
                        k: int, block: int, ws: Workspace, return_block_scores: bool = False):
    """Block-sparse baseline selection (mean-pooled block scores) -> indices [B, H, G, k]."""
    d = dims_of(Q, K)
    G = num_groups(d.n_q, group_size)
    idx = torch.empty((d.batch, d.heads, G, k), dtype=torch.int32, device=Q.device)
    bs = (torch.empty((d.batch, d.heads, G, d.n_kv // block), dtype=torch.float32,
                      device=Q.device) if return_block_scores else None)
    _check(lib().tlsp_pooled_block_select(ctypes.byref(d), _ptr(Q), _ptr(K), _ptr(groups),
                                          group_size, k, block, _ptr(idx), _ptr(bs), ws.ptr,
                                          ws.nbytes, _stream()),
           "tlsp_pooled_block_select")
    return (idx, bs) if return_block_scores else idx
