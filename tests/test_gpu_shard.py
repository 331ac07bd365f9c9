"""Head sharding through the CUDA library on one GPU.

Every step of the path is per head (grouping, scores, selection, both sparse
passes), so the heads of one batch element can be split over ranks with no
exchange. Here the shards run one after another on cuda:0: each shard's
inputs are the workload's own numbers for its heads, and every output of the
sharded calls (groups, indices, R, O_full and the reuse output) must equal the
unsharded call's output for the same head, bit for bit.
"""
import dataclasses

import pytest
import torch

from token_level_sparse_pddp_b200 import multi
from token_level_sparse_pddp_b200.synthetic import InputStream, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from token_level_sparse_pddp_b200 import build, tlsp
    build.build()
    return tlsp


def _run(T, wl, head_ids):
    """Anchor step then one reuse step of `wl` on the given heads."""
    it = iter(InputStream(wl, head_ids=head_ids, steps=2))
    _, _, Qa, Ka, Va = next(it)
    _, _, Qr, Kr, Vr = next(it)
    Qa, Ka, Va, Qr, Kr, Vr = (x.cuda() for x in (Qa, Ka, Va, Qr, Kr, Vr))
    gs, k = wl.group_size, wl.k
    ws = T.Workspace(T.dims_of(Qa, Ka), gs, k)
    groups = T.group_queries(Qa, gs, ws)
    O_full, idx, R = T.anchor_attention(Qa, Ka, Va, groups, gs, k, ws)
    O = T.reuse_attention(Qr, Kr, Vr, groups, gs, k, idx, R, ws)
    torch.cuda.synchronize()
    assert ws.status() == T.TLSP_OK
    return dict(groups=groups, idx=idx, R=R, O_full=O_full, O=O)


@pytest.mark.parametrize("wl_i,heads,world", [(1, 8, 2), (2, 4, 2), (2, 3, 2)])
def test_head_shards_equal_the_unsharded_call(T, wl_i, heads, world):
    # workload 1 (all 8 heads, 4 + 4) and the 32760-token workload on 4 heads
    # (2 + 2) and on 3 heads (an uneven 2 + 1 split)
    wl = dataclasses.replace(workload(wl_i), heads=heads)
    full = _run(T, wl, list(range(heads)))
    for rank in range(world):
        hs = list(multi.head_shard(heads, world, rank))
        part = _run(T, wl, hs)
        for name, ref in full.items():
            got = part[name]
            assert torch.equal(got, ref[:, hs[0]:hs[-1] + 1]), (name, rank, hs)
