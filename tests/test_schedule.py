"""The anchor / reuse schedule module: step decisions on CPU, and on the GPU the
same outputs as the explicit sequence of library calls."""
import pytest
import torch

from token_level_sparse_pddp_b200.schedule import MCSparseAttention
from token_level_sparse_pddp_b200.synthetic import InputStream, workload


def test_anchor_decisions():
    a = MCSparseAttention(16, 8, anchor_every=3)
    assert [a.is_anchor(s) for s in range(7)] == [True, False, False, True, False, False, True]
    b = MCSparseAttention(16, 8, schedule="ARAR")
    assert [b.is_anchor(s) for s in range(6)] == [True, False, True, False, True, False]
    with pytest.raises(ValueError):
        MCSparseAttention(16, 8, schedule="AX")
    with pytest.raises(ValueError):
        MCSparseAttention(0, 8)


@pytest.mark.gpu
def test_schedule_matches_explicit_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from token_level_sparse_pddp_b200 import build, tlsp
    build.build()
    wl = workload(1)
    gs, k = wl.group_size, wl.k
    attn = MCSparseAttention(gs, k, schedule=wl.schedule)
    ws = None
    state = {}
    for s, kind, Q, K, V in InputStream(wl):
        Q, K, V = Q.cuda(), K.cuda(), V.cuda()
        O = attn(Q, K, V)
        assert attn.last_was_anchor == (kind == "A")
        if ws is None:
            ws = tlsp.Workspace(tlsp.dims_of(Q, K), gs, k)
        if kind == "A":
            state["g"] = tlsp.group_queries(Q, gs, ws)
            ref, state["i"], state["R"] = tlsp.anchor_attention(Q, K, V, state["g"], gs, k, ws)
        else:
            ref = tlsp.reuse_attention(Q, K, V, state["g"], gs, k, state["i"], state["R"], ws)
        torch.cuda.synchronize()
        assert torch.equal(O, ref), s
    assert attn.status() == 0 and ws.status() == 0
    # a change of shape forces an anchor step
    Q2 = torch.zeros((1, 2, 256, 128), dtype=torch.bfloat16, device="cuda")
    attn(Q2, Q2, Q2)
    assert attn.last_was_anchor
