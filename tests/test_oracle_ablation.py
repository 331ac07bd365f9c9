"""Pins for the oracle's ablation functions (raster groups, block-granular and
mean-pooled block selection), checked against brute force, closed forms and the
token-level functions they reduce to."""
import itertools

import numpy as np
import pytest

from oracle import oracle as orc


def test_raster_groups_cover_in_order():
    g = orc.raster_groups(10, 4)
    assert g.tolist() == [0, 1, 2, 3, 4, 5, 6, 7, 8, 9, -1, -1]
    assert orc.raster_groups(8, 4).tolist() == list(range(8))


def test_block_topk_with_unit_blocks_is_token_topk():
    rng = np.random.default_rng(3)
    s = rng.standard_normal(64)
    for k in (1, 7, 64):
        assert np.array_equal(orc.block_topk(s, k, 1), orc.topk(s, k))


def test_block_topk_brute_force():
    """Among all kb-subsets of blocks exactly one beats every left-out block
    (higher sum, or equal sum and lower index); it must be the one chosen."""
    rng = np.random.default_rng(4)
    b, nb = 3, 6
    for trial in range(20):
        s = rng.integers(0, 4, size=b * nb).astype(float)  # many ties between block sums
        sums = s.reshape(nb, b).sum(1)
        for kb in range(1, nb + 1):
            ok = [c for c in itertools.combinations(range(nb), kb)
                  if all(sums[m] > sums[o] or (sums[m] == sums[o] and m < o)
                         for m in c for o in range(nb) if o not in c)]
            assert len(ok) == 1
            want = np.concatenate([np.arange(m * b, m * b + b) for m in ok[0]])
            assert np.array_equal(orc.block_topk(s, kb * b, b), want)


def test_block_sums_closed_form():
    s = np.arange(12, dtype=float)
    assert orc.block_sums(s, 4).tolist() == [6.0, 22.0, 38.0]


def test_pooled_scores_closed_form_and_selection():
    rng = np.random.default_rng(5)
    d, b, nb = 8, 4, 5
    K = rng.standard_normal((nb * b, d))
    Qg = rng.standard_normal((3, d))
    sc = orc.pooled_block_scores(Qg, K, b)
    for m in range(nb):
        want = np.dot(Qg.mean(0), K[m * b:(m + 1) * b].mean(0)) / np.sqrt(d)
        assert sc[m] == pytest.approx(want, rel=1e-14, abs=1e-14)
    # identical key rows inside a block: the pooled score equals the token score
    Kc = np.repeat(rng.standard_normal((nb, d)), b, axis=0)
    q1 = rng.standard_normal((1, d))
    tok = (Kc @ q1[0]) / np.sqrt(d)
    assert np.allclose(orc.pooled_block_scores(q1, Kc, b), tok[::b])
    sel = orc.pooled_block_select(Qg, K, 2 * b, b)
    best = np.sort(np.argsort(-sc, kind="stable")[:2])
    assert np.array_equal(sel, np.concatenate([np.arange(m * b, m * b + b) for m in best]))


def test_block_selection_with_all_keys_gives_dense_attention():
    rng = np.random.default_rng(6)
    Q, K, V = (rng.standard_normal((n, 16)) for n in (5, 24, 24))
    idx = orc.block_topk(rng.standard_normal(24), 24, 4)
    assert np.array_equal(idx, np.arange(24))
    O, _ = orc.dense(Q, K, V)
    assert np.allclose(orc.sparse(Q, K, V, idx), O, rtol=1e-13, atol=1e-13)


# ----------------------------------------------------------------- error decomposition

def _textbook_sparse_row(q, K, V, sel):
    """Softmax of q . K[sel] / sqrt(d) over the selected keys only, times V[sel]."""
    s = K[sel] @ q / np.sqrt(q.shape[0])
    p = np.exp(s - s.max())
    return (p / p.sum()) @ V[sel]


def test_rel_l2_closed_forms():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((2, 3, 5, 4))
    assert orc.rel_l2(x, x) == 0.0 and orc.rel_l2_head_mean(x, x) == 0.0
    assert abs(orc.rel_l2(2 * x, x) - 1.0) < 1e-12
    assert abs(orc.rel_l2_head_mean(-x, x) - 2.0) < 1e-12
    y = x.copy()
    y[1, 2] *= 3.0   # one head off by 2x its own norm
    assert abs(orc.rel_l2_head_mean(y, x) - 2.0 / 6) < 1e-12


def test_sparse_output_all_keys_is_dense_output():
    rng = np.random.default_rng(7)
    B, H, n, d, gs = 1, 2, 12, 8, 4
    Q, K, V = (rng.standard_normal((B, H, n, d)) for _ in range(3))
    groups = np.broadcast_to(orc.raster_groups(n, gs), (B, H, n)).copy()
    idx = np.broadcast_to(np.arange(n, dtype=np.int32), (B, H, n // gs, n)).copy()
    O_sp = orc.sparse_output(Q, K, V, groups, gs, idx)
    assert np.abs(O_sp - orc.dense_output(Q, K, V)).max() < 1e-12
    err = orc.decomposition(Q, K, V, [(groups, gs, idx)])
    assert err[0][0] < 1e-12 and err[0][1] < 1e-12


def test_sparse_output_matches_textbook_per_group():
    """Ragged grouping in a shuffled order, a different selection per group."""
    rng = np.random.default_rng(8)
    B, H, n, d, gs, k = 2, 1, 10, 6, 4, 5
    Q, K, V = (rng.standard_normal((B, H, n, d)) for _ in range(3))
    G = -(-n // gs)
    groups = np.full((B, H, G * gs), -1, dtype=np.int32)
    idx = np.empty((B, H, G, k), dtype=np.int32)
    for b in range(B):
        perm = rng.permutation(n)
        for g in range(G):
            members = np.sort(perm[g * gs:(g + 1) * gs])
            groups[b, 0, g * gs:g * gs + members.size] = members
            idx[b, 0, g] = np.sort(rng.choice(n, size=k, replace=False))
    O = orc.sparse_output(Q, K, V, groups, gs, idx)
    for b in range(B):
        for g in range(G):
            for t in orc.group_rows(groups[b, 0], gs, g):
                want = _textbook_sparse_row(Q[b, 0, t], K[b, 0], V[b, 0], idx[b, 0, g])
                assert np.abs(O[b, 0, t] - want).max() < 1e-12


def test_decomposition_per_query_selection_by_hand():
    """One query, two keys of three: the error is computed by hand from the
    textbook dense and sparse outputs."""
    q = np.array([[[[1.0, 0.0]]]])
    K = np.array([[[[1.0, 0.0], [0.0, 1.0], [-1.0, 0.0]]]])
    V = np.array([[[[1.0, 0.0], [0.0, 1.0], [0.0, 0.0]]]])
    s = np.array([1.0, 0.0, -1.0]) / np.sqrt(2)
    p = np.exp(s) / np.exp(s).sum()
    dense = p @ V[0, 0]
    p2 = np.exp(s[:2]) / np.exp(s[:2]).sum()
    sparse = p2 @ V[0, 0, :2]
    want = np.linalg.norm(sparse - dense) / np.linalg.norm(dense)
    groups = np.zeros((1, 1, 1), dtype=np.int32)
    idx = np.array([[[[0, 1]]]], dtype=np.int32)
    (got, got_h), = orc.decomposition(q, K, V, [(groups, 1, idx)])
    assert abs(got - want) < 1e-12 and abs(got_h - want) < 1e-12
