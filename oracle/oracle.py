"""fp64 CPU oracle for the MC-Sparse hot path: ctypes wrapper and step compositions.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the package smoke check and
by the benchmark's CPU-baseline / reference leg, never by the product path.
It shares no code with the CUDA library (it loads its own liboracle from
tlsp_oracle.cpp in this directory).

All array arguments are numpy arrays of one (batch, head) slice; they are
widened to float64 here (the bf16/fp32 values are represented exactly).
The compositions follow the anchor / reuse schedule of the MC-Sparse review
("Deconstructing and Closing the Dense-Sparse Attention Gap in Diffusion
Transformers", section 3): on an anchor step dense attention, exact group
scores, top-k selection, sparse attention and the residual R = O_full - O_sparse;
on a reuse step sparse attention over the cached selection plus R.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tlsp_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

N_ITER = 16  # power-iteration count (reading of "fast" PDDP: fixed, no convergence test)


def build(force: bool = False) -> str:
    """Compile the oracle's C++ into liboracle.so beside it (idempotent)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c++17",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, dp, fp, ip = ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
            lib.orc_dense_rows.argtypes = [i64, i64, i64, dp, dp, dp, dp, dp]
            lib.orc_group_scores.argtypes = [i64, i64, i64, dp, dp, dp, dp]
            lib.orc_topk.argtypes = [i64, dp, i64, ip]
            lib.orc_sparse_rows.argtypes = [i64, i64, dp, dp, dp, i64, ip, dp]
            lib.orc_pddp_direction.argtypes = [i64, ip, i64, dp, ctypes.c_int, dp, dp]
            lib.orc_pddp.argtypes = [i64, i64, dp, i64, ctypes.c_int, ip, dp, i64]
            lib.orc_pddp.restype = i64
            lib.orc_pddp_replay.argtypes = [i64, i64, i64, fp, ip, i64, dp, ctypes.c_int, dp]
            lib.orc_pddp_replay.restype = i64
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().float().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_levels(n: int, gs: int) -> int:
    g = -(-n // gs)
    return int(np.ceil(np.log2(g))) if g > 1 else 0


# ----------------------------------------------------------------- single steps

def dense(Q, K, V):
    """Dense attention of rows Q [m, d] over K, V [nkv, d] -> (O [m, d], LSE [m])."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    m, d = Q.shape
    O = np.empty((m, d)); L = np.empty(m)
    _load().orc_dense_rows(m, K.shape[0], d, _p(Q), _p(K), _p(V), _p(O), _p(L))
    return O, L


def group_scores(Qg, LSEg, K):
    """S [nkv]: summed exact softmax probability of the rows Qg on every key."""
    Qg, LSEg, K = _f64(Qg), _f64(LSEg), _f64(K)
    S = np.empty(K.shape[0])
    _load().orc_group_scores(Qg.shape[0], K.shape[0], K.shape[1], _p(Qg), _p(LSEg), _p(K), _p(S))
    return S


def topk(s, k: int) -> np.ndarray:
    """Ascending indices of the k largest entries of s (ties to the lower index)."""
    s = _f64(s)
    kk = min(int(k), s.shape[0])
    idx = np.empty(kk, dtype=np.int32)
    _load().orc_topk(s.shape[0], _p(s), k, _p(idx))
    return idx


def sparse(Q, K, V, idx):
    """Sparse attention of rows Q over the keys idx, softmax renormalised over idx."""
    Q, K, V, idx = _f64(Q), _f64(K), _f64(V), _i32(idx)
    m, d = Q.shape
    O = np.empty((m, d))
    _load().orc_sparse_rows(m, d, _p(Q), _p(K), _p(V), idx.shape[0], _p(idx), _p(O))
    return O


def pddp_direction(X, members=None, n_iter: int = N_ITER):
    """(mu, v): centre and leading principal direction of X[members]."""
    X = _f64(X)
    members = _i32(np.arange(X.shape[0]) if members is None else members)
    mu = np.empty(X.shape[1]); v = np.empty(X.shape[1])
    _load().orc_pddp_direction(members.shape[0], _p(members), X.shape[1], _p(X), n_iter, _p(mu), _p(v))
    return mu, v


def pddp(X, gs: int, n_iter: int = N_ITER, trace: bool = False):
    """PDDP grouping of one head's queries X [n, d] -> groups [G * gs] (-1 pads).

    With trace=True also returns the per-level projections [levels, n].
    """
    X = _f64(X)
    n, d = X.shape
    G = -(-n // gs)
    groups = np.empty(G * gs, dtype=np.int32)
    L = num_levels(n, gs)
    tr = np.empty((max(L, 1), n)) if trace else None
    got = _load().orc_pddp(n, d, _p(X), gs, n_iter, _p(groups), _p(tr) if trace else None, L)
    assert got == L, (got, L)
    return (groups, tr[:L]) if trace else groups


def pddp_replay(proj, n: int, gs: int, X=None, n_iter: int = N_ITER):
    """Groups obtained by cutting every node on the given fp32 projections [levels, n].

    If X is given, also returns this oracle's own fp64 projections on the very
    same nodes, for a numeric comparison of the supplied ones.
    """
    proj = np.ascontiguousarray(proj, dtype=np.float32)
    levels = proj.shape[0] if proj.ndim == 2 else 0
    G = -(-n // gs)
    groups = np.empty(G * gs, dtype=np.int32)
    own = None
    if X is not None:
        X = _f64(X)
        own = np.empty((max(levels, 1), n))
    got = _load().orc_pddp_replay(n, gs, levels, _p(proj), _p(groups),
                                  X.shape[1] if X is not None else 0,
                                  _p(X) if X is not None else None, n_iter,
                                  _p(own) if own is not None else None)
    assert got == num_levels(n, gs), (got, num_levels(n, gs))
    return (groups, own[:levels]) if X is not None else groups


# ------------------------------------------------------------- step compositions

def group_rows(groups, gs: int, g: int) -> np.ndarray:
    """Token ids of group g (padding dropped)."""
    rows = _i32(groups)[g * gs:(g + 1) * gs]
    return rows[rows >= 0]


def anchor_groups(Q, K, V, groups, gs: int, k: int, group_ids=None, O_full_stored=None):
    """Anchor step for some groups of one head.

    Returns a dict keyed by group id with rows, O_full [m, d], LSE [m], S [nkv],
    idx [k], O_sp [m, d], R [m, d]. R = O_full - O_sp, where O_full is the
    oracle's own fp64 dense output unless O_full_stored [n_q, d] (the dense
    output as another implementation stored it) is given.
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    G = -(-Q.shape[0] // gs)
    out = {}
    for g in (range(G) if group_ids is None else group_ids):
        rows = group_rows(groups, gs, g)
        Of, L = dense(Q[rows], K, V)
        S = group_scores(Q[rows], L, K)
        idx = topk(S, k)
        Osp = sparse(Q[rows], K, V, idx)
        base = Of if O_full_stored is None else _f64(O_full_stored)[rows]
        out[g] = dict(rows=rows, O_full=Of, LSE=L, S=S, idx=idx, O_sp=Osp, R=base - Osp)
    return out


def reuse_groups(Q, K, V, groups, gs: int, idx_by_group, R_by_group, group_ids=None):
    """Reuse step: O = sparse(current Q, K, V; anchor selection) + anchor R, per group."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    out = {}
    for g in (idx_by_group.keys() if group_ids is None else group_ids):
        rows = group_rows(groups, gs, g)
        out[g] = sparse(Q[rows], K, V, idx_by_group[g]) + _f64(R_by_group[g])
    return out


# ----------------------------------------------------------------- ablation
# The components MC-Sparse replaces (review section 3 and its ablation table:
# exact KV selection, token granularity, query grouping and residual
# compensation added one by one on top of block-sparse attention with
# mean-pooled scores). Plain numpy, fp64.

def raster_groups(n_q: int, gs: int) -> np.ndarray:
    """Query groups of consecutive tokens: group g = tokens g*gs .. g*gs + gs - 1, -1 past n_q."""
    G = -(-n_q // gs)
    q = np.arange(G * gs)
    return np.where(q < n_q, q, -1).astype(np.int32)


def select_blocks(block_scores, kb: int, b: int) -> np.ndarray:
    """The kb blocks of largest score (ties to the lower block, ascending), expanded to
    their b keys each (block m holds keys m*b .. m*b + b - 1), ascending."""
    blocks = topk(block_scores, kb)
    return (blocks.astype(np.int64)[:, None] * b + np.arange(b)[None, :]).ravel().astype(np.int32)


def block_sums(s, b: int) -> np.ndarray:
    """Block score of exact per-key scores: the sum over each block of b consecutive keys."""
    s = _f64(s)
    return s.reshape(-1, b).sum(axis=1)


def block_topk(s, k: int, b: int) -> np.ndarray:
    """Block-granular exact selection: k / b blocks by summed exact score, expanded."""
    return select_blocks(block_sums(s, b), k // b, b)


def pooled_block_scores(Qg, K, b: int) -> np.ndarray:
    """Block-sparse baseline scoring: mean of the group's query rows dotted with the
    mean of each block's key rows, scaled by 1/sqrt(d)."""
    Qg, K = _f64(Qg), _f64(K)
    d = K.shape[1]
    qbar = Qg.mean(axis=0)
    kbar = K.reshape(-1, b, d).mean(axis=1)
    return (kbar @ qbar) / np.sqrt(d)


def pooled_block_select(Qg, K, k: int, b: int) -> np.ndarray:
    """Block-sparse baseline selection: k / b blocks by mean-pooled score, expanded."""
    return select_blocks(pooled_block_scores(Qg, K, b), k // b, b)


# ----------------------------------------------------------------- error decomposition
# The review's account of the dense-sparse gap (section 2 and its Fig. 2): the
# sparse output differs from dense attention through the discarded tail (keys
# left out even by an exact per-query selection), structural binding (one
# selection shared by a query group, or by a key block) and selection error
# (approximate scores). Each rung below is one selection; its error is the
# relative L2 distance of the fp64 sparse output to the fp64 dense output.

def sparse_output(Q, K, V, groups, gs: int, idx) -> np.ndarray:
    """Sparse attention of every query of every head over its group's selection.

    Q [B, H, n_q, d], K, V [B, H, n_kv, d], groups [B, H, G*gs] (-1 padding),
    idx [B, H, G, k] -> O [B, H, n_q, d] in fp64 (no residual)."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    groups, idx = np.asarray(groups), np.asarray(idx)
    B, H, n_q, d = Q.shape
    O = np.zeros((B, H, n_q, d))
    G = -(-n_q // gs)
    for b in range(B):
        for h in range(H):
            for g in range(G):
                rows = group_rows(groups[b, h], gs, g)
                if rows.size:
                    O[b, h, rows] = sparse(Q[b, h][rows], K[b, h], V[b, h], idx[b, h, g])
    return O


def dense_output(Q, K, V) -> np.ndarray:
    """Dense attention of every query of every head -> O [B, H, n_q, d] in fp64."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    O = np.empty(Q.shape)
    for b in range(Q.shape[0]):
        for h in range(Q.shape[1]):
            O[b, h], _ = dense(Q[b, h], K[b, h], V[b, h])
    return O


def rel_l2(O, O_ref) -> float:
    """|O - O_ref| / |O_ref| over the whole tensor."""
    O, O_ref = _f64(O), _f64(O_ref)
    return float(np.linalg.norm(O - O_ref) / np.linalg.norm(O_ref))


def rel_l2_head_mean(O, O_ref) -> float:
    """Mean over (batch, head) of each head's relative L2 distance."""
    O, O_ref = _f64(O), _f64(O_ref)
    B, H = O.shape[:2]
    a, r = O.reshape(B, H, -1), O_ref.reshape(B, H, -1)
    return float((np.linalg.norm(a - r, axis=2) / np.linalg.norm(r, axis=2)).mean())


def decomposition(Q, K, V, rungs):
    """Errors of a ladder of selections against dense attention, in fp64.

    rungs: list of (groups [B, H, G*gs], gs, idx [B, H, G, k]) -> list of
    (rel_l2, rel_l2_head_mean), one per rung, in order."""
    O_dense = dense_output(Q, K, V)
    out = []
    for groups, gs, idx in rungs:
        O = sparse_output(Q, K, V, groups, gs, idx)
        out.append((rel_l2(O, O_dense), rel_l2_head_mean(O, O_dense)))
    return out
