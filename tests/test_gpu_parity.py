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
    wl = workload(4)
    assert_ok(run_and_compare(wl, sample_heads=[39], sample_groups=[5, 590], topk_rows=16,
                              replay_own=False))


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


def test_grouping_zero_spread_is_consecutive(T):
    n, gs = 100, 16
    Q = torch.ones((1, 2, n, 64), dtype=torch.bfloat16, device="cuda") * 0.375
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


def test_bounded_wait_times_out_and_context_survives(T):
    Q = torch.zeros((1, 1, 16, 64), device="cuda")
    ws = T.Workspace(T.dims_of(Q), 16, 1)
    T.debug_bounded_wait(ws, 2000)
    torch.cuda.synchronize()
    assert ws.status() == T.TLSP_ERR_TIMEOUT
    ws.reset()
    x = torch.arange(10, device="cuda").sum().item()   # context still usable
    assert x == 45 and ws.status() == T.TLSP_OK
