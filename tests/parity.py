"""GPU-vs-oracle parity helpers shared by the GPU tests and the smoke check.

The CUDA path runs through the C ABI (token_level_sparse_pddp_b200.tlsp); the
fp64 oracle (oracle/oracle.py) is fed the very same rounded inputs. Grouping
and top-k are compared bit-exactly with the oracle fed the GPU's own
projections / scores; attention outputs and residuals element by element
within the tolerance of the input precision (max-abs 2e-2 and mean-abs 2e-3
for bf16 inputs with fp32 accumulation, 1e-4 for fp32 inputs). Downstream
checks use the GPU's groups and indices on both sides, so output errors
measure arithmetic only.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np
import torch

from oracle import oracle as orc
from token_level_sparse_pddp_b200 import tlsp
from token_level_sparse_pddp_b200.synthetic import InputStream, Workload

TOL = {"f32": (1e-4, 1e-4), "bf16": (2e-2, 2e-3)}   # (max-abs, mean-abs)
SCORE_RTOL = {"f32": 1e-5, "bf16": 1e-3}           # |dS| / max_j S_g[j]


@dataclasses.dataclass
class Report:
    name: str
    errors: Dict[str, float] = dataclasses.field(default_factory=dict)
    info: Dict[str, float] = dataclasses.field(default_factory=dict)
    failures: List[str] = dataclasses.field(default_factory=list)

    def err(self, key, max_abs, mean_abs, tol):
        self.errors[key + ".max_abs"] = max(self.errors.get(key + ".max_abs", 0.0), max_abs)
        self.errors[key + ".mean_abs"] = max(self.errors.get(key + ".mean_abs", 0.0), mean_abs)
        if not (max_abs <= tol[0] and mean_abs <= tol[1]):
            self.failures.append(f"{key}: max_abs {max_abs:.3g} mean_abs {mean_abs:.3g} > {tol}")

    def check(self, ok: bool, what: str):
        if not ok:
            self.failures.append(what)


def _np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy() if t.dtype != torch.int32 else t.detach().cpu().numpy()


def check_group_structure(groups: np.ndarray, n: int, gs: int) -> Optional[str]:
    G = -(-n // gs)
    if groups.shape != (G * gs,):
        return "shape"
    real = groups[groups >= 0]
    if real.shape[0] != n or not np.array_equal(np.sort(real), np.arange(n)):
        return "not a partition of the queries"
    for g in range(G):
        blk = groups[g * gs:(g + 1) * gs]
        m = int((blk >= 0).sum())
        if m != (gs if g < G - 1 else n - (G - 1) * gs) or (blk[m:] != -1).any():
            return f"group {g} size"
        if (np.diff(blk[:m]) <= 0).any():
            return f"group {g} not ascending"
    return None


def run_and_compare(wl: Workload, sample_heads=None, sample_groups=None, topk_rows=None,
                    replay_own=True, steps=None, k=None, gs=None, stream=None) -> Report:
    """Runs the workload's schedule on the GPU and compares against the oracle.

    sample_heads / sample_groups restrict the oracle side (None = all);
    topk_rows caps the rows of the fed top-k check per head (None = all).
    """
    k = wl.k if k is None else k
    gs = wl.group_size if gs is None else gs
    rep = Report(wl.name)
    tol = TOL[wl.dtype]
    dev = torch.device("cuda")
    ws = None
    state = None
    heads = list(range(wl.heads)) if sample_heads is None else list(sample_heads)
    for step, kind, Q, K, V in InputStream(wl, steps=steps):
        Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
        if ws is None:
            ws = tlsp.Workspace(tlsp.dims_of(Qd, Kd), gs, k)
        n_q, n_kv = Q.shape[2], K.shape[2]
        G = -(-n_q // gs)
        if kind == "A":
            groups_d, proj_d = tlsp.group_queries(Qd, gs, ws, trace=True)
            O_d, idx_d, R_d, S_d = tlsp.anchor_attention(Qd, Kd, Vd, groups_d, gs, k, ws,
                                                         return_scores=True)
            torch.cuda.synchronize()
            rep.check(ws.status() == 0, f"device status {ws.status()} after anchor step {step}")
            groups = _np(groups_d)
            proj = proj_d.cpu().numpy()
            state = dict(groups=groups, idx={}, R={})
            for b in range(wl.batch):
                for h in range(wl.heads):
                    msg = check_group_structure(groups[b, h], n_q, gs)
                    rep.check(msg is None, f"groups b{b} h{h}: {msg}")
            for b in range(wl.batch):
                for h in heads:
                    X = Q[b, h].double().numpy()
                    fed = orc.pddp_replay(proj[:, b, h], n_q, gs, X=X if replay_own else None)
                    fed_groups = fed[0] if replay_own else fed
                    rep.check(np.array_equal(fed_groups, groups[b, h]),
                              f"groups b{b} h{h} differ from the oracle cut on the GPU projections")
                    if replay_own and proj.shape[0] > 0:
                        own = fed[1]
                        scale = max(np.abs(own).max(), 1e-30)
                        e = np.abs(own - proj[:, b, h]).max() / scale
                        rep.errors["proj.rel_max"] = max(rep.errors.get("proj.rel_max", 0), e)
                        rep.check(e <= (1e-4 if wl.dtype == "f32" else 2e-3),
                                  f"projections b{b} h{h}: rel err {e:.3g}")
                    if n_q <= 20000:
                        own_groups = orc.pddp(X, gs)
                        agree = np.mean(own_groups == groups[b, h])
                        rep.info["groups_e2e_agreement.min"] = min(
                            rep.info.get("groups_e2e_agreement.min", 1.0), float(agree))
            S_all = S_d.cpu().numpy()
            idx_all = _np(idx_d)
            O_full = _np(O_d)
            R_all = R_d.cpu().numpy()
            for b in range(wl.batch):
                for h in heads:
                    rows_chk = range(G) if topk_rows is None else np.unique(
                        np.linspace(0, G - 1, min(topk_rows, G)).astype(int))
                    for g in rows_chk:
                        fed = orc.topk(S_all[b, h, g].astype(np.float64), k)
                        if not np.array_equal(fed, idx_all[b, h, g]):
                            rep.failures.append(f"indices b{b} h{h} g{g} differ from fed top-k")
                    gsel = range(G) if sample_groups is None else sorted(
                        set(int(x) % G for x in sample_groups))
                    Xq, Xk, Xv = (T[b, h].double().numpy() for T in (Q, K, V))
                    for g in gsel:
                        rows = orc.group_rows(groups[b, h], gs, g)
                        Of, L = orc.dense(Xq[rows], Xk, Xv)
                        d_of = np.abs(O_full[b, h, rows] - Of)
                        rep.err("O_full", d_of.max(), d_of.mean(), tol)
                        S = orc.group_scores(Xq[rows], L, Xk)
                        es = np.abs(S_all[b, h, g] - S).max() / S.max()
                        rep.errors["scores.rel_max"] = max(rep.errors.get("scores.rel_max", 0), es)
                        rep.check(es <= SCORE_RTOL[wl.dtype], f"scores b{b} h{h} g{g}: {es:.3g}")
                        own_idx = orc.topk(S, k)
                        ov = len(np.intersect1d(own_idx, idx_all[b, h, g])) / k
                        rep.info["topk_overlap_vs_fp64.min"] = min(
                            rep.info.get("topk_overlap_vs_fp64.min", 1.0), ov)
                        Osp = orc.sparse(Xq[rows], Xk, Xv, idx_all[b, h, g])
                        R_ref = O_full[b, h, rows].astype(np.float64) - Osp
                        d_r = np.abs(R_all[b, h, rows] - R_ref)
                        rep.err("R", d_r.max(), d_r.mean(), tol)
                        state["idx"][(b, h, g)] = idx_all[b, h, g]
                        state["R"][(b, h, g)] = R_ref
        else:
            assert state is not None, "schedule must start with an anchor step"
            groups_d = torch.from_numpy(state["groups"]).to(dev)
            O_d = tlsp.reuse_attention(Qd, Kd, Vd, groups_d, gs, k, idx_d, R_d, ws)
            torch.cuda.synchronize()
            rep.check(ws.status() == 0, f"device status {ws.status()} after reuse step {step}")
            O = _np(O_d)
            for (b, h, g), idx in state["idx"].items():
                rows = orc.group_rows(state["groups"][b, h], gs, g)
                Xq, Xk, Xv = (T[b, h].double().numpy() for T in (Q, K, V))
                ref = orc.sparse(Xq[rows], Xk, Xv, idx) + state["R"][(b, h, g)]
                d_o = np.abs(O[b, h, rows] - ref)
                rep.err("O_reuse", d_o.max(), d_o.mean(), tol)
    return rep
