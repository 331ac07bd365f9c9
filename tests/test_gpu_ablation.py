"""GPU parity of the ablation kernels (raster groups, block-granular selection,
mean-pooled block selection) through the C ABI against the fp64 oracle."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from tests.parity import TOL
from token_level_sparse_pddp_b200.synthetic import InputStream, Workload, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from token_level_sparse_pddp_b200 import build, tlsp
    build.build()
    return tlsp


@pytest.mark.parametrize("n_q,gs", [(128, 16), (1000, 64), (32760, 128), (5, 8)])
def test_raster_groups_bit_exact(T, n_q, gs):
    Q = torch.zeros((2, 3, n_q, 64), dtype=torch.bfloat16, device="cuda")
    g = T.group_raster(Q, gs).cpu().numpy()
    want = orc.raster_groups(n_q, gs)
    for b in range(2):
        for h in range(3):
            assert np.array_equal(g[b, h], want)


@pytest.mark.parametrize("rows,n_kv,k,b", [(37, 1024, 256, 64), (8, 32760, 1664, 104),
                                           (5, 96, 96, 8), (4, 64, 16, 1), (3, 48, 48, 48)])
def test_block_topk_fed_same_scores(T, rows, n_kv, k, b):
    g = torch.Generator().manual_seed(rows * 7 + b)
    # integer-valued scores: many ties between block sums, sums exact in fp32
    s = torch.randint(0, 5, (rows, n_kv), generator=g).float().cuda()
    idx, bs = T.block_topk_from_scores(s, k, b, return_block_scores=True)
    idx, bs, sn = idx.cpu().numpy(), bs.cpu().numpy(), s.cpu().numpy()
    for r in range(rows):
        assert np.array_equal(bs[r], orc.block_sums(sn[r], b))           # exact: integer sums
        assert np.array_equal(idx[r], orc.block_topk(sn[r], k, b))
    if b == 1:
        assert np.array_equal(idx, T.topk_from_scores(s, k).cpu().numpy())


def test_block_topk_real_scores(T):
    """Exact group scores of a real anchor step, blocked: the GPU block sums match the
    oracle's fp64 sums of the same fp32 scores, and the selection is bit-exact when the
    oracle is fed the GPU's block sums."""
    wl = workload(1)
    _, _, Q, K, V = next(iter(InputStream(wl, steps=1)))
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    ws = T.Workspace(T.dims_of(Qd, Kd), wl.group_size, wl.k)
    groups = T.group_queries(Qd, wl.group_size, ws)
    _, _, _, S = T.anchor_attention(Qd, Kd, Vd, groups, wl.group_size, wl.k, ws, return_scores=True)
    idx, bs = T.block_topk_from_scores(S, wl.k, 64, return_block_scores=True)
    S, idx, bs = S.cpu().numpy(), idx.cpu().numpy(), bs.cpu().numpy()
    for h in range(wl.heads):
        for g in range(S.shape[2]):
            want = orc.block_sums(S[0, h, g].astype(np.float64), 64)
            assert np.abs(bs[0, h, g] - want).max() <= 1e-5 * max(want.max(), 1e-30)
            assert np.array_equal(idx[0, h, g], orc.select_blocks(bs[0, h, g], wl.k // 64, 64))


def _pooled_case(T, wl, b, raster):
    _, _, Q, K, V = next(iter(InputStream(wl, steps=1)))
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    gs, k = wl.group_size, wl.k
    ws = T.Workspace(T.dims_of(Qd, Kd), gs, k)
    groups = T.group_raster(Qd, gs) if raster else T.group_queries(Qd, gs, ws)
    idx, bs = T.pooled_block_select(Qd, Kd, groups, gs, k, b, ws, return_block_scores=True)
    torch.cuda.synchronize()
    assert ws.status() == 0
    return Q, K, V, Qd, Kd, Vd, ws, groups, idx, bs


@pytest.mark.parametrize("wl_i,b,raster", [(0, 16, True), (0, 8, False), (1, 64, True),
                                           (1, 32, False)])
def test_pooled_block_select(T, wl_i, b, raster):
    wl = workload(wl_i)
    Q, K, V, Qd, Kd, Vd, ws, groups, idx, bs = _pooled_case(T, wl, b, raster)
    gs = wl.group_size
    G = -(-wl.n_q // gs)
    g_np, idx, bs = groups.cpu().numpy(), idx.cpu().numpy(), bs.cpu().numpy()
    for bb in range(wl.batch):
        for h in range(wl.heads):
            Kh = K[bb, h].double().numpy()
            for g in range(G):
                rows = orc.group_rows(g_np[bb, h], gs, g)
                want = orc.pooled_block_scores(Q[bb, h].double().numpy()[rows], Kh, b)
                scale = max(np.abs(want).max(), 1e-30)
                assert np.abs(bs[bb, h, g] - want).max() <= 1e-4 * scale
                assert np.array_equal(idx[bb, h, g],
                                      orc.select_blocks(bs[bb, h, g], wl.k // b, b))


def test_block_sparse_baseline_output(T):
    """Block-sparse baseline end to end: pooled block selection, then the library's
    sparse pass with no residual (R = 0), against the oracle's sparse attention over
    the same keys."""
    wl = workload(1)
    Q, K, V, Qd, Kd, Vd, ws, groups, idx, bs = _pooled_case(T, wl, 64, True)
    R0 = torch.zeros(Qd.shape, dtype=torch.float32, device="cuda")
    O = T.reuse_attention(Qd, Kd, Vd, groups, wl.group_size, wl.k, idx, R0, ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    O, g_np, idx = O.float().cpu().numpy(), groups.cpu().numpy(), idx.cpu().numpy()
    max_abs, mean_abs = TOL[wl.dtype]
    errs = []
    for h in range(wl.heads):
        Qh, Kh, Vh = (X[0, h].double().numpy() for X in (Q, K, V))
        for g in range(0, -(-wl.n_q // wl.group_size), 3):
            rows = orc.group_rows(g_np[0, h], wl.group_size, g)
            want = orc.sparse(Qh[rows], Kh, Vh, idx[0, h, g])
            errs.append(np.abs(O[0, h][rows] - want))
    e = np.concatenate([x.ravel() for x in errs])
    assert e.max() <= max_abs and e.mean() <= mean_abs, (e.max(), e.mean())


def test_block_selection_all_keys_equals_dense(T):
    """k = n_kv with any block size selects every key: the sparse pass equals dense."""
    wl = Workload("blk-all", 1, 2, 128, (2, 8, 8), None, "bf16", 16, 128, "A", 0.0, 11)
    Q, K, V, Qd, Kd, Vd, ws, groups, idx, bs = _pooled_case(T, wl, 32, True)
    assert np.array_equal(idx.cpu().numpy()[0, 0, 0], np.arange(128))
    R0 = torch.zeros(Qd.shape, dtype=torch.float32, device="cuda")
    O = T.reuse_attention(Qd, Kd, Vd, groups, wl.group_size, wl.k, idx, R0, ws)
    Od = T.dense_attention(Qd, Kd, Vd, ws)
    torch.cuda.synchronize()
    assert (O.float() - Od.float()).abs().max().item() <= 2e-2


def test_ablation_runner_structure(T):
    from token_level_sparse_pddp_b200 import ablation
    wl = workload(1)
    rows = ablation.run(wl, 64)
    kinds = {(r["step"], r["variant"]): r for r in rows}
    assert len(rows) == len(wl.schedule) * len(ablation.VARIANTS)
    for r in rows:
        assert np.isfinite(r["rel_l2"]) and r["ms"] > 0
        if r["kind"] == "A":  # dense pass on anchor steps: the output is the dense output
            assert r["rel_l2"] == 0.0
    # the bsa variant is sparse on every step, including the anchor steps
    assert kinds[(0, "bsa")]["rel_l2"] > 0.0


def test_ablation_all_keys_is_dense(T):
    from token_level_sparse_pddp_b200 import ablation
    wl = Workload("abl-all", 1, 2, 128, (2, 8, 8), None, "bf16", 16, 128, "ARR", 0.05, 13)
    for r in ablation.run(wl, 32):
        assert r["rel_l2"] <= 5e-3, r


def test_error_decomposition_structure(T):
    """Each rung adds an error source; with every key selected all rungs are dense."""
    from token_level_sparse_pddp_b200 import ablation
    rows = ablation.decompose(workload(1), 64)
    assert [r["component"] for r in rows] == [c for c, _ in ablation.DECOMPOSITION]
    assert all(np.isfinite(r["rel_l2"]) and r["rel_l2"] > 0 for r in rows)
    wl = Workload("dec-all", 1, 2, 128, (2, 8, 8), None, "bf16", 16, 128, "A", 0.0, 17)
    for r in ablation.decompose(wl, 32):
        assert r["rel_l2"] <= 5e-3, r


def test_error_decomposition_matches_the_oracle(T):
    """Workload 1, every group of every head: the oracle's fp64 outputs on the
    GPU runner's own selections give the same rel-L2 per rung (the GPU side is
    bf16 attention with fp32 accumulation)."""
    from oracle import oracle as orc
    from token_level_sparse_pddp_b200 import ablation
    rows, (Q, K, V), sels = ablation.decompose(workload(1), 64, return_selections=True)
    ref = orc.decomposition(Q.double().numpy(), K.double().numpy(), V.double().numpy(), sels)
    for r, (e, e_h) in zip(rows, ref):
        print(r["component"], r["rel_l2"], e, r["rel_l2_head_mean"], e_h)
        assert abs(r["rel_l2"] - e) <= 2e-3 + 1e-2 * e, (r, e)
        assert abs(r["rel_l2_head_mean"] - e_h) <= 2e-3 + 1e-2 * e_h, (r, e_h)


def test_recomputed_selection_variant(T):
    """The per-step recomputed selection: on every reuse step its selection is
    bit-exactly the oracle's top-k fed that step's own exact scores, and it
    differs from the anchor's cached one (the inputs drift)."""
    from oracle import oracle as orc
    from token_level_sparse_pddp_b200 import ablation
    wl = workload(1)
    rec = {}
    rows = ablation.run(wl, 64, record=rec)
    assert sorted(rec) == [s for s, kind in enumerate(wl.schedule) if kind != "A"]
    for s, r in rec.items():
        S, idx = r["S"].cpu().numpy(), r["idx"].cpu().numpy()
        for b in range(S.shape[0]):
            for h in range(S.shape[1]):
                for g in range(S.shape[2]):
                    assert np.array_equal(orc.topk(S[b, h, g].astype(np.float64), wl.k),
                                          idx[b, h, g]), (s, b, h, g)
    by = {(r["step"], r["variant"]): r for r in rows}
    for s in rec:
        assert by[(s, "recompute_token")]["rel_l2"] > 0
        assert by[(s, "recompute_token")]["rel_l2"] != by[(s, "pddp_token")]["rel_l2"]

