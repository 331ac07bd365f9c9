"""Pins of the fp64 oracle against things other than itself.

Each test checks one oracle function against a textbook routine (numpy
softmax, numpy.linalg.eigh, lexsort), a closed form, brute force on tiny
inputs, an invariant the definitions imply, or a case worked by hand
(tests/golden). The definitions followed are those of the MC-Sparse review
("Deconstructing and Closing the Dense-Sparse Attention Gap in Diffusion
Transformers", section 3 "Method & Key Results").
"""
import itertools
import json
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def textbook_attention(Q, K, V):
    s = Q @ K.T / np.sqrt(Q.shape[1])
    s = s - s.max(axis=1, keepdims=True)
    P = np.exp(s)
    P /= P.sum(axis=1, keepdims=True)
    return P @ V, P


def rand(rng, *shape):
    return rng.standard_normal(shape)


# ------------------------------------------------------------------ dense attention

def test_dense_matches_textbook_softmax(orc):
    rng = np.random.default_rng(11)
    Q, K, V = rand(rng, 37, 64), rand(rng, 53, 64), rand(rng, 53, 64)
    O, L = orc.dense(Q, K, V)
    O_ref, P = textbook_attention(Q, K, V)
    np.testing.assert_allclose(O, O_ref, rtol=0, atol=1e-12)
    # LSE is the log partition function: exp(s - LSE) sums to one per row.
    s = Q @ K.T / 8.0
    np.testing.assert_allclose(np.exp(s - L[:, None]).sum(axis=1), 1.0, atol=1e-12)
    np.testing.assert_allclose(np.exp(s - L[:, None]), P, atol=1e-13)


def test_dense_on_first_workload_inputs(orc):
    from token_level_sparse_pddp_b200.synthetic import InputStream, workload
    _, _, Q, K, V = next(iter(InputStream(workload(0))))
    for h in range(Q.shape[1]):
        q, k, v = (x[0, h].double().numpy() for x in (Q, K, V))
        O, _ = orc.dense(q, k, v)
        np.testing.assert_allclose(O, textbook_attention(q, k, v)[0], atol=1e-12)


def test_dense_identical_keys_is_mean_of_values(orc):
    # All keys equal -> every logit equal -> uniform weights: O = mean(V), LSE = s + ln n.
    rng = np.random.default_rng(3)
    d, n = 16, 40
    Q = rand(rng, 5, d)
    k = rand(rng, d)
    K = np.tile(k, (n, 1))
    V = rand(rng, n, d)
    O, L = orc.dense(Q, K, V)
    np.testing.assert_allclose(O, np.tile(V.mean(axis=0), (5, 1)), atol=1e-13)
    np.testing.assert_allclose(L, Q @ k / 4.0 + np.log(n), atol=1e-13)


def test_golden_two_key_example(orc):
    g = json.load(open(os.path.join(GOLDEN, "attention_2keys.json")))
    Q, K, V = (np.array(g[x]) for x in ("Q", "K", "V"))
    O, L = orc.dense(Q, K, V)
    np.testing.assert_allclose(O, g["O_full"], atol=1e-12)
    np.testing.assert_allclose(L, g["LSE"], atol=1e-12)
    S = orc.group_scores(Q, L, K)
    np.testing.assert_allclose(S, g["S"], atol=1e-12)
    idx = orc.topk(S, g["k"])
    assert idx.tolist() == g["idx"]
    Osp = orc.sparse(Q, K, V, idx)
    np.testing.assert_allclose(Osp, g["O_sp"], atol=1e-12)
    res = orc.anchor_groups(Q, K, V, np.array([0]), 1, g["k"])[0]
    np.testing.assert_allclose(res["R"], g["R"], atol=1e-12)


# ------------------------------------------------------------------ group scores

def test_scores_sum_to_group_size_and_nonnegative(orc):
    rng = np.random.default_rng(5)
    Q, K = rand(rng, 24, 32), rand(rng, 70, 32)
    _, L = orc.dense(Q, K, K)
    S = orc.group_scores(Q[:24], L[:24], K)
    assert (S >= 0).all()
    assert abs(S.sum() - 24) < 1e-11


def test_scores_single_query_is_probability_row(orc):
    rng = np.random.default_rng(6)
    Q, K, V = rand(rng, 3, 32), rand(rng, 50, 32), rand(rng, 50, 32)
    _, L = orc.dense(Q, K, V)
    _, P = textbook_attention(Q, K, V)
    for r in range(3):
        np.testing.assert_allclose(orc.group_scores(Q[r:r + 1], L[r:r + 1], K), P[r], atol=1e-14)


def test_scores_are_summed_probability_rows(orc):
    rng = np.random.default_rng(7)
    Q, K, V = rand(rng, 30, 16), rand(rng, 45, 16), rand(rng, 45, 16)
    _, L = orc.dense(Q, K, V)
    _, P = textbook_attention(Q, K, V)
    rows = np.array([2, 5, 7, 11, 29])
    np.testing.assert_allclose(orc.group_scores(Q[rows], L[rows], K), P[rows].sum(axis=0), atol=1e-13)


# ------------------------------------------------------------------ top-k

@pytest.mark.parametrize("seed", range(20))
def test_topk_matches_lexsort_with_ties(orc, seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 60))
    s = rng.integers(0, 6, size=n).astype(np.float64)  # many ties
    k = int(rng.integers(1, n + 1))
    order = np.lexsort((np.arange(n), -s))  # primary: value descending, then index ascending
    assert orc.topk(s, k).tolist() == sorted(order[:k].tolist())


def test_topk_brute_force_tiny(orc):
    # Over all 0/1/2-valued vectors of length 6 and every k: the chosen set has
    # the largest score sum, and among sets with that sum the smallest index sum.
    for vals in itertools.product([0.0, 1.0, 2.0], repeat=6):
        s = np.array(vals)
        for k in range(1, 7):
            best = min(itertools.combinations(range(6), k),
                       key=lambda c: (-s[list(c)].sum(), sum(c)))
            assert orc.topk(s, k).tolist() == list(best)


def test_topk_full_and_negative_zero(orc):
    s = np.array([0.0, -0.0, 0.0, 1.0])
    assert orc.topk(s, 4).tolist() == [0, 1, 2, 3]
    assert orc.topk(s, 2).tolist() == [0, 3]  # -0 ties +0: lower index wins
    assert orc.topk(s, 10).tolist() == [0, 1, 2, 3]


# ------------------------------------------------------------------ sparse attention

def test_sparse_with_all_keys_is_dense(orc):
    rng = np.random.default_rng(8)
    Q, K, V = rand(rng, 9, 32), rand(rng, 41, 32), rand(rng, 41, 32)
    np.testing.assert_allclose(orc.sparse(Q, K, V, np.arange(41)),
                               textbook_attention(Q, K, V)[0], atol=1e-12)


def test_sparse_is_softmax_over_selected_columns(orc):
    rng = np.random.default_rng(9)
    Q, K, V = rand(rng, 9, 32), rand(rng, 41, 32), rand(rng, 41, 32)
    idx = np.array([1, 4, 5, 17, 30, 40])
    np.testing.assert_allclose(orc.sparse(Q, K, V, idx),
                               textbook_attention(Q, K[idx], V[idx])[0], atol=1e-12)


def test_anchor_identity_and_zero_drift_reuse(orc):
    rng = np.random.default_rng(10)
    n, d, gs, k = 64, 16, 8, 12
    Q, K, V = rand(rng, n, d), rand(rng, n, d), rand(rng, n, d)
    groups = orc.pddp(Q, gs)
    anc = orc.anchor_groups(Q, K, V, groups, gs, k)
    O_dense = textbook_attention(Q, K, V)[0]
    for g, a in anc.items():
        np.testing.assert_allclose(a["O_sp"] + a["R"], a["O_full"], atol=1e-13)
        np.testing.assert_allclose(a["O_full"], O_dense[a["rows"]], atol=1e-12)
    reu = orc.reuse_groups(Q, K, V, groups, gs, {g: a["idx"] for g, a in anc.items()},
                           {g: a["R"] for g, a in anc.items()})
    for g in anc:
        np.testing.assert_allclose(reu[g], O_dense[anc[g]["rows"]], atol=1e-12)


def test_full_selection_gives_zero_residual(orc):
    rng = np.random.default_rng(12)
    n, d, gs = 40, 16, 8
    Q, K, V = rand(rng, n, d), rand(rng, n, d), rand(rng, n, d)
    groups = orc.pddp(Q, gs)
    for g, a in orc.anchor_groups(Q, K, V, groups, gs, n).items():
        assert a["idx"].tolist() == list(range(n))
        np.testing.assert_allclose(a["R"], 0.0, atol=1e-13)


# ------------------------------------------------------------------ PDDP grouping

def check_structure(groups, n, gs):
    G = -(-n // gs)
    assert groups.shape == (G * gs,)
    real = groups[groups >= 0]
    assert sorted(real.tolist()) == list(range(n))  # disjoint and covering
    for g in range(G):
        blk = groups[g * gs:(g + 1) * gs]
        m = int((blk >= 0).sum())
        assert m == (gs if g < G - 1 else n - (G - 1) * gs)
        assert (blk[m:] == -1).all()  # padding only at the end of the last group
        assert (np.diff(blk[:m]) > 0).all()  # ascending inside a group


@pytest.mark.parametrize("n,gs", [(128, 16), (37, 4), (100, 7), (64, 64), (5, 8), (1, 1), (75, 1)])
def test_pddp_structure(orc, n, gs):
    rng = np.random.default_rng(n * 31 + gs)
    X = rand(rng, n, 6)
    groups = orc.pddp(X, gs)
    check_structure(groups, n, gs)


def test_pddp_golden_line(orc):
    g = json.load(open(os.path.join(GOLDEN, "pddp_line_2d.json")))
    assert orc.pddp(np.array(g["X"]), g["group_size"]).tolist() == g["groups"]


@pytest.mark.parametrize("sign", [1.0, -1.0])
@pytest.mark.parametrize("n,gs", [(37, 4), (64, 8), (50, 5)])
def test_pddp_points_on_a_line(orc, sign, n, gs):
    # Collinear points: every node's principal direction is the line direction,
    # so the grouping is "sort by position along the line, cut into chunks of
    # gs" with the direction oriented so its largest component is positive.
    rng = np.random.default_rng(n)
    d = 8
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    u *= np.sign(u[np.argmax(np.abs(u))]) * sign
    t = rng.permutation(n).astype(np.float64) + rng.uniform(0, 0.5, n)
    X = np.outer(t, u) + rng.standard_normal(d)
    order = np.argsort(t if sign > 0 else -t)
    G = -(-n // gs)
    expect = np.full(G * gs, -1)
    for g in range(G):
        chunk = np.sort(order[g * gs:(g + 1) * gs])
        expect[g * gs:g * gs + len(chunk)] = chunk
    assert orc.pddp(X, gs).tolist() == expect.tolist()


def test_pddp_zero_spread_splits_by_index(orc):
    # All queries equal: no principal direction, every projection is 0 and
    # the cut falls to the token index -> consecutive runs.
    n, gs = 30, 4
    X = np.tile(np.arange(5.0), (n, 1))
    G = -(-n // gs)
    expect = [i if i < n else -1 for i in range(G * gs)]
    assert orc.pddp(X, gs).tolist() == expect


def test_pddp_direction_matches_eigh(orc):
    # Clear eigengap: the fixed 16 power iterations reach the top eigenvector
    # of the centred covariance (numpy.linalg.eigh) to 1e-9.
    rng = np.random.default_rng(13)
    n, d = 60, 10
    scales = np.array([5.0, 1.5] + [1.0] * (d - 2))
    R, _ = np.linalg.qr(rng.standard_normal((d, d)))
    X = (rng.standard_normal((n, d)) * scales) @ R.T + 3.0
    mu, v = orc.pddp_direction(X)
    np.testing.assert_allclose(mu, X.mean(axis=0), atol=1e-13)
    C = X - X.mean(axis=0)
    w, E = np.linalg.eigh(C.T @ C)
    top = E[:, -1]
    top *= np.sign(top[np.argmax(np.abs(top))])
    assert abs(abs(v @ top) - 1) < 1e-9
    np.testing.assert_allclose(v, top, atol=1e-5)


def test_pddp_split_brute_force(orc):
    # N = 8, gs = 4: the root cut must be, among all C(8,4) balanced
    # bipartitions, the one whose left half has the smallest sum of
    # projections on the exact principal direction (eigh), i.e. the rank cut.
    for seed in range(10):
        rng = np.random.default_rng(100 + seed)
        X = rng.standard_normal((8, 3)) * np.array([4.0, 1.0, 0.5])
        groups = orc.pddp(X, 4)
        C = X - X.mean(axis=0)
        _, E = np.linalg.eigh(C.T @ C)
        v = E[:, -1] * np.sign(E[np.argmax(np.abs(E[:, -1])), -1])
        p = C @ v
        best = min(itertools.combinations(range(8), 4), key=lambda c: p[list(c)].sum())
        assert groups[:4].tolist() == sorted(best)
        assert groups[4:].tolist() == sorted(set(range(8)) - set(best))


def test_pddp_replay_closed_forms(orc):
    n, gs = 37, 4
    L = orc.num_levels(n, gs)
    G = -(-n // gs)
    ids = np.arange(n, dtype=np.float32)
    # Projection = +token id at every level: consecutive runs.
    up = orc.pddp_replay(np.tile(ids, (L, 1)), n, gs)
    assert up.tolist() == [i if i < n else -1 for i in range(G * gs)]
    # Projection = -token id: every cut sends the highest ids left, the ragged
    # right chain keeps the lowest ones -> runs of descending blocks, token 0 last.
    down = orc.pddp_replay(np.tile(-ids, (L, 1)), n, gs)
    expect = []
    for g in range(G - 1):
        expect += list(range(n - gs * (g + 1), n - gs * g))
    rest = n - gs * (G - 1)
    expect += list(range(rest)) + [-1] * (gs - rest)
    assert down.tolist() == expect


def test_pddp_replay_of_own_trace(orc):
    rng = np.random.default_rng(14)
    X = rng.standard_normal((100, 12))
    groups, tr = orc.pddp(X, 8, trace=True)
    again, own = orc.pddp_replay(tr.astype(np.float32), 100, 8, X=X)
    np.testing.assert_allclose(own, tr, atol=1e-12)
    # fp32 rounding of the projections may only swap exact near-ties; there are none here.
    assert again.tolist() == groups.tolist()


def test_num_levels():
    from oracle.oracle import num_levels
    assert [num_levels(n, 1) for n in (1, 2, 3, 4, 5, 8, 9)] == [0, 1, 2, 2, 3, 3, 4]
    assert num_levels(32760, 128) == 8 and num_levels(75600, 128) == 10 and num_levels(4680, 128) == 6
