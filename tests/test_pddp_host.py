"""Host-side invariants of the PDDP tree that the CUDA library sizes its
shared memory by (no GPU needed).

A node at offset `off` with `cnt` tokens and `slots` leaf slots sends
floor(slots/2)*gs tokens left (the rank cut of fast PDDP, MC-Sparse review
section 3). The library stages a node's order keys in shared memory with room
for ceil(n_q / 2^level) + gs keys at each level (the split kernels and the
levels finished inside the direction kernel), so every node of a level must
fit that bound; and the leaves must tile [0, n_q) with G - 1 full groups."""
import math
import random

import pytest


def _tree(n_q: int, gs: int):
    G = (n_q + gs - 1) // gs
    L = 0
    while (1 << L) < G:
        L += 1
    nodes = [(0, n_q, G)]
    per_level = []
    for _ in range(L):
        per_level.append([n for n in nodes if n[2] > 1])
        nxt = []
        for off, cnt, slots in nodes:
            if slots > 1:
                ls = slots // 2
                nxt += [(off, ls * gs, ls), (off + ls * gs, cnt - ls * gs, slots - ls)]
            else:
                nxt.append((off, cnt, slots))
        nodes = nxt
    return G, per_level, nodes


def _cases():
    rnd = random.Random(7)
    fixed = [(32760, 128), (75600, 128), (4680, 128), (1024, 64), (128, 16), (1, 16),
             (129, 128), (65536, 256), (100001, 32)]
    return fixed + [(rnd.randint(1, 300000), rnd.choice([16, 32, 64, 128, 256]))
                    for _ in range(400)]


@pytest.mark.parametrize("n_q,gs", _cases()[:9])
def test_fixed_shapes(n_q, gs):
    _check(n_q, gs)


def test_random_shapes():
    for n_q, gs in _cases()[9:]:
        _check(n_q, gs)


def _check(n_q, gs):
    G, per_level, leaves = _tree(n_q, gs)
    for level, nodes in enumerate(per_level):
        bound = math.ceil(n_q / (1 << level)) + gs
        assert all(cnt <= bound for _, cnt, _ in nodes), (n_q, gs, level)
        assert all(slots > 1 and cnt > (slots - 1) * gs for _, cnt, slots in nodes)
    assert len(leaves) == G and all(slots == 1 for _, _, slots in leaves)
    assert [off for off, _, _ in leaves] == [g * gs for g in range(G)]
    assert all(cnt == gs for _, cnt, _ in leaves[:-1])
    assert 1 <= leaves[-1][1] <= gs
