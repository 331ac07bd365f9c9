"""Ablation of MC-Sparse on the library's own kernels.

    python -m token_level_sparse_pddp_b200.ablation [--workload I] [--block B] [--steps S]
    python -m token_level_sparse_pddp_b200.ablation --decompose [--workload I] [--heads H]

The MC-Sparse review (section 3 and its ablation table) builds the method from
block-sparse attention with mean-pooled scores by adding, one at a time, exact KV
selection, token granularity, query grouping and residual compensation. This
runs that ladder at equal density (k keys per query group) on a workload's
synthetic schedule and prints, per step and variant, the relative L2 error of the
output against the library's dense attention (|O - O_dense| / |O_dense| over the
whole [B, H, n_q, d] tensor, and its mean over heads) and the device time of the
step's selection and sparse work:

  bsa           raster query groups, mean-pooled block scores recomputed every
                step, block-granular selection, no residual;
  exact_block   raster groups, exact scores on anchor steps (selection cached for
                the reuse steps), block-granular selection, no residual;
  exact_token   as exact_block with token-level selection;
  pddp_token    as exact_token with PDDP query groups;
  recompute_token
                as pddp_token, but the exact token selection is made again on
                every step from that step's own exact scores (the groups are
                still the anchor's): set against pddp_token on the reuse steps
                it isolates what reusing an anchor's selection costs in error
                (the review's case for reuse is the temporal stability of the
                selections) and what recomputing it costs in time;
  mc_sparse     as pddp_token with the dense-sparse residual R added back.

On an anchor step every variant except bsa runs the dense pass anyway (exact
scores need it), so its output there is the dense output and the error is 0.
Every step runs through the C ABI; nothing here computes attention itself.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
from typing import Dict, List

import torch

from . import tlsp
from .synthetic import InputStream, workload

VARIANTS = ("bsa", "exact_block", "exact_token", "pddp_token", "recompute_token", "mc_sparse")


def rel_l2(O: torch.Tensor, O_ref: torch.Tensor) -> float:
    a, r = O.float(), O_ref.float()
    return float(torch.linalg.vector_norm(a - r) / torch.linalg.vector_norm(r))


def rel_l2_head_mean(O: torch.Tensor, O_ref: torch.Tensor) -> float:
    """Mean over (batch, head) of each head's relative L2 error: heads whose dense
    output is small (diffuse attention) weigh as much as the others."""
    a, r = O.float().flatten(2), O_ref.float().flatten(2)
    return float((torch.linalg.vector_norm(a - r, dim=2) /
                  torch.linalg.vector_norm(r, dim=2)).mean())


def run(wl, block: int, steps: int = 0, record: Dict = None) -> List[Dict]:
    """The ladder on the workload's schedule. With `record` (a dict), the
    recompute_token variant's groups, selection and exact scores of every
    reuse step are kept in it under the step number."""
    if wl.n_kv % block or wl.k % block:
        raise ValueError(f"block {block} must divide n_kv={wl.n_kv} and k={wl.k}")
    dev = torch.device("cuda")
    gs, k = wl.group_size, wl.k
    rows = []
    ws = None
    state: Dict[str, Dict] = {v: {} for v in VARIANTS}

    def timed(fn):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        out = fn()
        b.record()
        torch.cuda.synchronize()
        return out, a.elapsed_time(b)

    for s, kind, Q, K, V in InputStream(wl, steps=steps or None):
        Q, K, V = Q.to(dev), K.to(dev), V.to(dev)
        if ws is None:
            ws = tlsp.Workspace(tlsp.dims_of(Q, K), gs, k)
            raster = tlsp.group_raster(Q, gs)
            R0 = torch.zeros(Q.shape, dtype=torch.float32, device=dev)
        O_dense = tlsp.dense_attention(Q, K, V, ws)
        torch.cuda.synchronize()
        for v in VARIANTS:
            st = state[v]
            if v == "bsa":
                def step():
                    idx = tlsp.pooled_block_select(Q, K, raster, gs, k, block, ws)
                    return tlsp.reuse_attention(Q, K, V, raster, gs, k, idx, R0, ws)
                O, ms = timed(step)
            elif v == "recompute_token" and kind != "A":
                def step():
                    _, idx, _, S = tlsp.anchor_attention(Q, K, V, st["groups"], gs, k, ws,
                                                         return_scores=True)
                    return tlsp.reuse_attention(Q, K, V, st["groups"], gs, k, idx, R0, ws), idx, S
                (O, idx, S), ms = timed(step)
                if record is not None:
                    record[s] = dict(groups=st["groups"], idx=idx, S=S)
                del S
            elif kind == "A":
                def step():
                    groups = raster if v in ("exact_block", "exact_token") else \
                        tlsp.group_queries(Q, gs, ws)
                    O_full, idx, R, S = tlsp.anchor_attention(Q, K, V, groups, gs, k, ws,
                                                              return_scores=True)
                    if v == "exact_block":
                        idx = tlsp.block_topk_from_scores(S, k, block)
                    return O_full, groups, idx, R
                (O, groups, idx, R), ms = timed(step)
                st.update(groups=groups, idx=idx, R=R if v == "mc_sparse" else R0)
            else:
                O, ms = timed(lambda: tlsp.reuse_attention(Q, K, V, st["groups"], gs, k,
                                                           st["idx"], st["R"], ws))
            if ws.status() != 0:
                raise RuntimeError(f"device status {tlsp.status_string(ws.status())} in {v}")
            rows.append(dict(step=s, kind=kind if v != "bsa" else "S", variant=v,
                             rel_l2=rel_l2(O, O_dense),
                             rel_l2_head_mean=rel_l2_head_mean(O, O_dense), ms=ms))
    return rows


DECOMPOSITION = (
    ("tail", "per-query exact token selection (discarded tail only)"),
    ("query_binding", "+ one selection per PDDP query group (exact, token level)"),
    ("kv_binding", "+ block-granular selection (exact block scores)"),
    ("selection", "+ approximate scoring (mean-pooled block scores)"),
    ("bsa", "+ raster query groups (block-sparse attention)"),
)


def decompose(wl, block: int, return_selections: bool = False):
    """The review's three sparse-attention errors (structural binding, selection,
    discarded tail) taken apart on the first step of a workload: each row adds one
    source of error to the one before and reports the rel-L2 of the sparse output
    (no residual) against dense attention. Per-query selection is the library's
    grouping with group size 1. With return_selections, also returns the
    inputs (Q, K, V on the host) and each rung's (groups, group size,
    selection) on the host, so the same selections can be evaluated elsewhere."""
    if wl.n_kv % block or wl.k % block:
        raise ValueError(f"block {block} must divide n_kv={wl.n_kv} and k={wl.k}")
    dev = torch.device("cuda")
    _, _, Q, K, V = next(iter(InputStream(wl, steps=1)))
    Q, K, V = Q.to(dev), K.to(dev), V.to(dev)
    gs, k = wl.group_size, wl.k
    ws1 = tlsp.Workspace(tlsp.dims_of(Q, K), 1, k)
    ws = tlsp.Workspace(tlsp.dims_of(Q, K), gs, k)
    O_dense = tlsp.dense_attention(Q, K, V, ws)
    R0 = torch.zeros(Q.shape, dtype=torch.float32, device=dev)
    out = []

    sels = []

    def sparse(groups, g, idx, w):
        if return_selections:
            sels.append((groups.cpu().numpy(), g, idx.cpu().numpy()))
        return tlsp.reuse_attention(Q, K, V, groups, g, k, idx, R0, w)

    single = tlsp.group_raster(Q, 1)
    _, idx1, _ = tlsp.anchor_attention(Q, K, V, single, 1, k, ws1)
    out.append(sparse(single, 1, idx1, ws1))
    del ws1, idx1
    pddp = tlsp.group_queries(Q, gs, ws)
    _, idx, _, S = tlsp.anchor_attention(Q, K, V, pddp, gs, k, ws, return_scores=True)
    out.append(sparse(pddp, gs, idx, ws))
    out.append(sparse(pddp, gs, tlsp.block_topk_from_scores(S, k, block), ws))
    del S
    out.append(sparse(pddp, gs, tlsp.pooled_block_select(Q, K, pddp, gs, k, block, ws), ws))
    raster = tlsp.group_raster(Q, gs)
    out.append(sparse(raster, gs, tlsp.pooled_block_select(Q, K, raster, gs, k, block, ws), ws))
    torch.cuda.synchronize()
    if ws.status() != 0:
        raise RuntimeError(f"device status {tlsp.status_string(ws.status())}")
    rows = [dict(component=c, what=w, rel_l2=rel_l2(O, O_dense),
                 rel_l2_head_mean=rel_l2_head_mean(O, O_dense))
            for (c, w), O in zip(DECOMPOSITION, out)]
    if return_selections:
        return rows, (Q.cpu(), K.cpu(), V.cpu()), sels
    return rows


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", type=int, default=1)
    ap.add_argument("--block", type=int, default=0,
                    help="key block size (default: 64 for workloads 0-1, 104 for 2)")
    ap.add_argument("--steps", type=int, default=0, help="steps of the schedule (0 = all)")
    ap.add_argument("--heads", type=int, default=0, help="run with only this many heads")
    ap.add_argument("--decompose", action="store_true",
                    help="error decomposition on the first step instead of the ladder")
    args = ap.parse_args()
    wl = workload(args.workload)
    if args.heads:
        wl = dataclasses.replace(wl, heads=args.heads, name=f"{wl.name}-H{args.heads}")
    block = args.block or {0: 16, 1: 64, 2: 104}.get(args.workload, 64)
    rows = decompose(wl, block) if args.decompose else run(wl, block, args.steps)
    for r in rows:
        print(json.dumps(dict(workload=wl.name, block=block, k=wl.k, **r)), flush=True)


if __name__ == "__main__":
    main()
