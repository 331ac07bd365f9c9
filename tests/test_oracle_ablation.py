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
