"""GPU parity when the rows of one warp disagree about raising the softmax
reference max.

Both attention kernels keep a reference max per query row and raise it (and
rescale what was accumulated against the old one) only when a block of scores
exceeds it by more than 2^8. Here a few keys carry large logits for a subset of
the queries only (every 2nd, 4th or 8th row), placed so that raises happen:
inside a warpgroup's first chunk, in later chunks (rescaling O and the P blocks
already written), twice for the same rows, and in the ragged last chunk's
neighbourhood. Outputs and log partitions are compared with the fp64 oracle on
the same bf16 inputs.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from tests.parity import TOL

N_Q, N_KV, D, H = 256, 552, 128, 2  # 2 query tiles; 4 full key chunks + a ragged one
# (key, channel, rows, key value): those rows get q[channel] = 8, so their logit on
# the key is 8 * value / sqrt(128) nats, 28-42 nats above everything else
SPIKES = ((70, 3, lambda i: i % 8 == 5, 45.0),
          (228, 2, lambda i: i % 4 == 3, 50.0),
          (300, 0, lambda i: i % 2 == 1, 40.0),
          (450, 1, lambda i: i % 4 == 1, 60.0))


@pytest.fixture(scope="module")
def T():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from token_level_sparse_pddp_b200 import build, tlsp
    build.build()
    return tlsp


def _inputs():
    g = torch.Generator().manual_seed(5)
    Q = torch.randn(1, H, N_Q, D, generator=g) * 0.5
    K = torch.randn(1, H, N_KV, D, generator=g) * 0.5
    V = torch.randn(1, H, N_KV, D, generator=g)
    i = torch.arange(N_Q)
    for key, c, rows, val in SPIKES:
        Q[:, :, rows(i), c] = 8.0
        K[:, :, key, c] = val
    return Q.bfloat16(), K.bfloat16(), V.bfloat16()


def _log2_logits(Q, K):
    """fp64 logits of the bf16 inputs in log2 units, [H, n_q, n_kv]."""
    q, k = Q[0].double().numpy(), K[0].double().numpy()
    return np.einsum("hqd,hkd->hqk", q, k) / np.sqrt(D) / np.log(2.0)


def test_inputs_raise_in_part_of_each_warp():
    """The inputs do what the GPU tests need: in the dense pass (chunks of 128 keys
    in order) and in the sparse pass (the selection below), some rows of a warp
    exceed their running reference by more than 2^8 in a later chunk while other
    rows of the same warp do not."""
    Q, K, _ = _inputs()
    x = _log2_logits(Q, K)
    sel = np.union1d(np.arange(0, N_KV, 2), np.arange(1, 217, 2))
    for keys in (np.arange(N_KV), sel):
        xs = x[:, :, keys]
        ref = xs[:, :, :128].max(axis=2)          # reference after the first chunk
        mixed = 0
        for c0 in range(128, keys.shape[0], 128):
            cm = xs[:, :, c0:c0 + 128].max(axis=2)
            raise_ = cm > ref + 8.0
            for w in range(N_Q // 32):
                rows = slice(32 * w, 32 * (w + 1))
                r = raise_[:, rows]
                mixed += int((r.any(axis=1) & ~r.all(axis=1)).sum())
                # a warp that raises moves every row's reference to max(ref, chunk max)
                ref[:, rows] = np.where(r.any(axis=1, keepdims=True),
                                        np.maximum(ref[:, rows], cm[:, rows]), ref[:, rows])
        assert mixed > 0
    # and inside the first chunk, after its first 32-column block, for some rows only
    first = x[:, :, :128]
    late = first[:, :, 32:].max(axis=2) > first[:, :, :32].max(axis=2) + 8.0
    assert late.any() and not late.all()


@pytest.mark.gpu
def test_dense_partial_warp_raises(T):
    Q, K, V = _inputs()
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    ws = T.Workspace(T.dims_of(Qd, Kd), 128, 128)
    lse = torch.empty((1, H, N_Q), dtype=torch.float32, device="cuda")
    O = T.dense_attention(Qd, Kd, Vd, ws, lse=lse)
    torch.cuda.synchronize()
    assert ws.status() == 0
    O, lse = O.float().cpu().numpy(), lse.cpu().numpy()
    max_abs, mean_abs = TOL["bf16"]
    for h in range(H):
        want, L = orc.dense(Q[0, h].double().numpy(), K[0, h].double().numpy(),
                            V[0, h].double().numpy())
        # the spikes dominate the rows they hit (else the test would not raise)
        hit = np.arange(N_Q) % 2 == 1
        assert (L[hit] > L[~hit].max() + 10).all()
        e = np.abs(O[0, h] - want)
        assert e.max() <= max_abs and e.mean() <= mean_abs, (h, e.max(), e.mean())
        assert np.abs(lse[0, h] - L).max() <= 1e-3, (h, np.abs(lse[0, h] - L).max())


@pytest.mark.gpu
def test_sparse_partial_warp_raises(T):
    """The gathered pass over a selection that holds the spike keys in its chunks
    0-2 (positions 70, 222, 258, 333)."""
    Q, K, V = _inputs()
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    gs, k = 128, 384
    sel = np.union1d(np.arange(0, N_KV, 2), np.arange(1, 217, 2)).astype(np.int32)
    assert sel.shape[0] == k and all(s[0] in sel for s in SPIKES)
    ws = T.Workspace(T.dims_of(Qd, Kd), gs, k)
    groups = T.group_raster(Qd, gs)
    G = N_Q // gs
    idx = torch.from_numpy(np.broadcast_to(sel, (1, H, G, k)).copy()).cuda()
    R0 = torch.zeros(Qd.shape, dtype=torch.float32, device="cuda")
    O = T.reuse_attention(Qd, Kd, Vd, groups, gs, k, idx, R0, ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    O, g_np = O.float().cpu().numpy(), groups.cpu().numpy()
    max_abs, mean_abs = TOL["bf16"]
    for h in range(H):
        Qh, Kh, Vh = (X[0, h].double().numpy() for X in (Q, K, V))
        for g in range(G):
            rows = orc.group_rows(g_np[0, h], gs, g)
            e = np.abs(O[0, h][rows] - orc.sparse(Qh[rows], Kh, Vh, sel))
            assert e.max() <= max_abs and e.mean() <= mean_abs, (h, g, e.max(), e.mean())
