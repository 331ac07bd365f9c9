"""GPU parity: the CUDA path through the C ABI against the fp64 oracle."""
import numpy as np
import pytest
import torch

from tests.parity import check_group_structure, run_and_compare
from token_level_sparse_pddp_b200.synthetic import Workload, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from token_level_sparse_pddp_b200 import build, tlsp
    build.build()
    return tlsp


def assert_ok(rep):
    print(rep.name, rep.errors, rep.info)
    assert not rep.failures, rep.failures[:10]


def small(name, **kw):
    base = dict(name=name, batch=1, heads=2, head_dim=128, grid=(2, 8, 8), q_frames=None,
                dtype="bf16", group_size=16, k=32, schedule="ARR", drift=0.05, seed=7)
    base.update(kw)
    return Workload(**base)


# ------------------------------------------------------------ the five workloads

def test_workload0_tiny_fp32_full(T):
    assert_ok(run_and_compare(workload(0)))


def test_workload1_bf16_full(T):
    assert_ok(run_and_compare(workload(1)))


@pytest.mark.slow
def test_workload2_wan_sampled(T):
    wl = workload(2)
    assert_ok(run_and_compare(wl, sample_heads=[0, 11], sample_groups=[0, 77, 255],
                              topk_rows=64, replay_own=True))


@pytest.mark.slow
def test_workload3_ar_chunk_sampled(T):
    wl = workload(3)
    assert_ok(run_and_compare(wl, sample_heads=[3], sample_groups=[0, 36], topk_rows=37))


@pytest.mark.slow
def test_workload4_large_sampled(T):
    # two heads: the 10-level PDDP tree (591 groups, nodes down to 2 slots)
    # replayed against the oracle's fp64 projections, fed top-k on 64 rows per
    # head, outputs on sampled groups including the ragged last one
    wl = workload(4)
    rep = run_and_compare(wl, sample_heads=[0, 39], sample_groups=[5, 300, 590], topk_rows=64,
                          replay_own=True)
    assert_ok(rep)
    assert rep.errors["proj.rel_max"] <= 2e-3


# ------------------------------------------------------------ edge cases

@pytest.mark.parametrize("wl", [
    small("ragged-bf16", grid=(1, 10, 10), group_size=16, k=20),           # 100 = 6*16 + 4
    small("ragged-fp32-d64", grid=(1, 10, 10), head_dim=64, dtype="f32"),
    small("one-group", grid=(1, 6, 8), group_size=64, k=48),                # G = 1, k = n_kv
    small("k-equals-nkv", group_size=32, k=128),
    small("k-one", k=1),
    small("gs-one", grid=(1, 4, 8), group_size=1, k=8, schedule="AR"),
    small("nq-neq-nkv", grid=(4, 8, 8), q_frames=(2, 3), k=40),
    small("d64-bf16", head_dim=64, group_size=32, k=64),
    small("gs-not-pow2", grid=(3, 7, 9), group_size=24, k=50),
    small("batch2", batch=2, heads=3, grid=(2, 4, 8), group_size=8, k=16),
])
def test_edge_workloads(T, wl):
    assert_ok(run_and_compare(wl))


def test_k_equals_nkv_residual_vanishes(T):
    from token_level_sparse_pddp_b200.synthetic import InputStream
    wl = small("full-k", k=128, group_size=32)
    _, _, Q, K, V = next(iter(InputStream(wl)))
    Q, K, V = Q.cuda(), K.cuda(), V.cuda()
    ws = T.Workspace(T.dims_of(Q, K), 32, 128)
    groups = T.group_queries(Q, 32, ws)
    O, idx, R = T.anchor_attention(Q, K, V, groups, 32, 128, ws)
    assert (idx.cpu() == torch.arange(128, dtype=torch.int32)).all()
    # R = O_full (rounded to bf16) - O_sparse(all keys): only the bf16 rounding of O_full is left
    assert R.abs().max().item() <= 2.0 ** -8 * max(1.0, O.float().abs().max().item())


def test_topk_fed_ties_and_signed_zero(T):
    from oracle import oracle as orc
    rng = np.random.default_rng(0)
    for n_kv, k in [(1, 1), (7, 3), (100, 100), (1000, 37), (5000, 4999), (33000, 1664)]:
        S = rng.integers(0, 5, size=(6, n_kv)).astype(np.float32)
        S[0] = 0.0
        S[1, ::2] = -0.0
        S[2] = rng.standard_normal(n_kv).astype(np.float32)
        idx = T.topk_from_scores(torch.from_numpy(S).cuda(), k).cpu().numpy()
        for r in range(6):
            assert np.array_equal(idx[r], orc.topk(S[r].astype(np.float64), k)), (n_kv, k, r)


def test_topk_fed_many_rows_and_shapes(T):
    # more rows than the persistent grid (each CTA takes several rows), row
    # lengths that are not a multiple of 4, attention-like heavy-tailed rows
    # (the candidate-list path) and flat rows (the streaming fallback)
    from oracle import oracle as orc
    rng = np.random.default_rng(5)
    for rows, n_kv, k in [(700, 4096, 205), (9, 4095, 200), (12, 32760, 1664), (4, 75600, 7552),
                          (3, 130, 64)]:
        S = rng.exponential(1.0, size=(rows, n_kv)).astype(np.float32) ** 3
        S[0] = rng.standard_normal(n_kv).astype(np.float32)
        S[1] = 1.0                       # every key tied
        S[2, : n_kv // 2] = 0.5          # half the row tied, inside the selection's bin
        idx = T.topk_from_scores(torch.from_numpy(S).cuda(), k).cpu().numpy()
        check = range(rows) if rows <= 16 else list(range(8)) + list(range(rows - 8, rows))
        for r in check:
            assert np.array_equal(idx[r], orc.topk(S[r].astype(np.float64), k)), (n_kv, k, r)


def test_topk_structured_rows(T):
    # rows of 8K-64K keys with structure: a smooth field, sparse spikes, a
    # ramp, ties at the k-th key, a third of the row at the max, signed zeros;
    # every row must match the oracle
    from oracle import oracle as orc
    rng = np.random.default_rng(11)
    for rows, n_kv, k in [(600, 32760, 1664), (8, 8192, 300), (8, 65536, 2000), (9, 20001, 1000)]:
        S = rng.exponential(1.0, size=(rows, n_kv)).astype(np.float32) ** 3
        S[0] = np.cumsum(rng.standard_normal(n_kv)).astype(np.float32)   # smooth field
        S[1] = 0.0
        S[1, 63::64] = 1.0 + rng.random(len(S[1, 63::64])).astype(np.float32)  # sparse spikes
        S[2] = np.arange(n_kv, dtype=np.float32)[::-1]                       # ramp
        S[3] = np.round(S[3] * 4) / 4                                        # ties at the k-th key
        S[4, ::3] = S[4].max()                                               # a third of the row at the max
        S[5, 1::2] = -0.0
        S[5, ::2] = 0.0
        S[6] = rng.standard_normal(n_kv).astype(np.float32)
        idx = T.topk_from_scores(torch.from_numpy(S).cuda(), k).cpu().numpy()
        check = range(rows) if rows <= 16 else list(range(10)) + list(range(rows - 10, rows))
        for r in check:
            assert np.array_equal(idx[r], orc.topk(S[r].astype(np.float64), k)), (n_kv, k, r)


def test_split_fed_with_ties(T):
    from oracle import oracle as orc
    rng = np.random.default_rng(1)
    for n, n_left in [(1, 0), (1, 1), (10, 5), (999, 500), (4096, 128), (40000, 20000)]:
        members = np.sort(rng.choice(2 * n, size=n, replace=False)).astype(np.int32)
        proj = rng.integers(-3, 4, size=2 * n).astype(np.float32)
        proj[::7] = -0.0
        left, right = T.split_from_projections(torch.from_numpy(proj).cuda(),
                                               torch.from_numpy(members).cuda(), n_left)
        order = sorted(members.tolist(), key=lambda t: (float(proj[t]), t))
        assert left.cpu().tolist() == sorted(order[:n_left])
        assert right.cpu().tolist() == sorted(order[n_left:])


@pytest.mark.parametrize("n,d", [(100, 64), (100, 128), (3000, 128)])
def test_grouping_zero_spread_is_consecutive(T, n, d):
    # identical rows: every node has zero scatter, its direction is e_0 and
    # every projection ties, so each cut keeps token order (d = 128 takes the
    # tensor-core scatter and power iteration, 3000 rows its chunked levels)
    gs = 16
    Q = torch.ones((1, 2, n, d), dtype=torch.bfloat16, device="cuda") * 0.375
    ws = T.Workspace(T.dims_of(Q), gs, 1)
    groups = T.group_queries(Q, gs, ws).cpu().numpy()
    G = -(-n // gs)
    expect = [i if i < n else -1 for i in range(G * gs)]
    for h in range(2):
        assert groups[0, h].tolist() == expect
        assert check_group_structure(groups[0, h], n, gs) is None


def test_out_of_range_index_sets_device_status(T):
    from token_level_sparse_pddp_b200.synthetic import InputStream
    wl = small("bad-index")
    _, _, Q, K, V = next(iter(InputStream(wl)))
    Q, K, V = Q.cuda(), K.cuda(), V.cuda()
    ws = T.Workspace(T.dims_of(Q, K), 16, 32)
    groups = T.group_queries(Q, 16, ws)
    O, idx, R = T.anchor_attention(Q, K, V, groups, 16, 32, ws)
    torch.cuda.synchronize()
    assert ws.status() == T.TLSP_OK
    idx[0, 1, 3, 5] = 10 ** 6   # checked by the kernel before any use; the key is skipped
    T.reuse_attention(Q, K, V, groups, 16, 32, idx, R, ws)
    torch.cuda.synchronize()
    assert ws.status() == T.TLSP_ERR_DEVICE_ASSERT
    ws.reset()
    torch.cuda.synchronize()
    assert ws.status() == T.TLSP_OK


def _anchor_state(T, wl, gs, k):
    from token_level_sparse_pddp_b200.synthetic import InputStream
    it = iter(InputStream(wl))
    _, _, Q, K, V = next(it)
    _, _, Q1, K1, V1 = next(it)
    Q, K, V, Q1, K1, V1 = (x.cuda() for x in (Q, K, V, Q1, K1, V1))
    ws = T.Workspace(T.dims_of(Q, K), gs, k)
    groups = T.group_queries(Q, gs, ws)
    O, idx, R = T.anchor_attention(Q, K, V, groups, gs, k, ws)
    torch.cuda.synchronize()
    assert ws.status() == T.TLSP_OK
    return ws, groups, idx, R, (Q1, K1, V1)


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_negative_index_sets_device_status_and_spares_other_tiles(T, dtype, d):
    # a negative selection entry is caller-kept state gone bad: the kernel
    # records it before use, and every other group's output is unchanged
    wl = small("neg-index", dtype=dtype, head_dim=d, grid=(2, 8, 10))   # 160 queries, ragged tail
    gs, k = 16, 32
    ws, groups, idx, R, (Q1, K1, V1) = _anchor_state(T, wl, gs, k)
    clean = T.reuse_attention(Q1, K1, V1, groups, gs, k, idx, R, ws)
    bad = idx.clone()
    bad[0, 1, 3, 7] = -5
    out = T.reuse_attention(Q1, K1, V1, groups, gs, k, bad, R, ws)
    torch.cuda.synchronize()
    assert ws.status() == T.TLSP_ERR_DEVICE_ASSERT
    rows = groups[0, 1, 3 * gs:4 * gs].long()
    keep = torch.ones(out.shape[2], dtype=torch.bool, device=out.device)
    keep[rows[rows >= 0]] = False
    assert torch.equal(out[0, 0], clean[0, 0])
    assert torch.equal(out[0, 1][keep], clean[0, 1][keep])
    ws.reset()
    torch.cuda.synchronize()
    assert ws.status() == T.TLSP_OK


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_bad_group_entries_set_device_status(T, dtype, d):
    # -1 is padding only in the ragged tail of the last group; a -1 among a
    # full group's members, or a token id in the tail, is recorded
    wl = small("bad-group", dtype=dtype, head_dim=d, grid=(2, 8, 10))   # G = 10, last holds 16
    gs, k = 16, 32
    wl2 = small("bad-group-ragged", dtype=dtype, head_dim=d, grid=(3, 5, 10))  # 150 = 9*16 + 6
    for w, plant in ((wl, (0, 1, 5 * 16 + 5, -1)), (wl2, (0, 0, 9 * 16 + 10, 3))):
        ws, groups, idx, R, (Q1, K1, V1) = _anchor_state(T, w, gs, k)
        T.reuse_attention(Q1, K1, V1, groups, gs, k, idx, R, ws)
        torch.cuda.synchronize()
        assert ws.status() == T.TLSP_OK
        b, h, pos, val = plant
        bad = groups.clone()
        bad[b, h, pos] = val
        T.reuse_attention(Q1, K1, V1, bad, gs, k, idx, R, ws)
        torch.cuda.synchronize()
        assert ws.status() == T.TLSP_ERR_DEVICE_ASSERT, (w.name, plant)


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_reuse_needs_only_the_status_word(T, dtype, d):
    wl = small("reuse-ws", dtype=dtype, head_dim=d)
    gs, k = 16, 32
    ws, groups, idx, R, (Q1, K1, V1) = _anchor_state(T, wl, gs, k)
    full = T.reuse_attention(Q1, K1, V1, groups, gs, k, idx, R, ws)
    tiny = T.Workspace.status_only()
    assert tiny.nbytes == 256
    out = T.reuse_attention(Q1, K1, V1, groups, gs, k, idx, R, tiny)
    torch.cuda.synchronize()
    assert tiny.status() == T.TLSP_OK
    assert torch.equal(out, full)


def test_bounded_wait_times_out_and_context_survives(T):
    Q = torch.zeros((1, 1, 16, 64), device="cuda")
    ws = T.Workspace(T.dims_of(Q), 16, 1)
    T.debug_bounded_wait(ws, 2000)
    torch.cuda.synchronize()
    assert ws.status() == T.TLSP_ERR_TIMEOUT
    ws.reset()
    x = torch.arange(10, device="cuda").sum().item()   # context still usable
    assert x == 45 and ws.status() == T.TLSP_OK
