"""The dense-attention entry point that allocates nothing.

Some callers cannot allocate device memory or hand over a workspace (code
running while a CUDA graph is captured, or under a framework whose memory
pool owns all allocations). tlsp_dense_attention_noalloc serves them from a
fixed scratch array inside the library. This file checks, through the C ABI,
that it returns what tlsp_dense_attention returns, on two calls in a row,
that sampled rows agree with the fp64 oracle's dense attention, and that
requests larger than its fixed scratch are refused. It is named so that
pytest collects it last.
"""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

TOL = {torch.float32: (1e-4, 1e-4), torch.bfloat16: (2e-2, 2e-3)}  # (max-abs, mean-abs)


@pytest.fixture(scope="module")
def T():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from token_level_sparse_pddp_b200 import build, tlsp
    build.build()
    return tlsp


@pytest.mark.parametrize("dtype,B,H,n_q,n_kv,d", [
    (torch.bfloat16, 1, 4, 1000, 777, 128),
    (torch.bfloat16, 2, 3, 256, 4096, 128),
    (torch.float32, 1, 2, 128, 200, 64),
])
def test_noalloc_matches_workspace_entry_point(T, dtype, B, H, n_q, n_kv, d):
    g = torch.Generator(device="cuda").manual_seed(n_q + n_kv)
    Q = torch.randn((B, H, n_q, d), generator=g, device="cuda").to(dtype)
    K = torch.randn((B, H, n_kv, d), generator=g, device="cuda").to(dtype)
    V = torch.randn((B, H, n_kv, d), generator=g, device="cuda").to(dtype)
    ws = T.Workspace(T.dims_of(Q, K), 1, 1)
    ref = T.dense_attention(Q, K, V, ws)
    max_tol, mean_tol = TOL[dtype]
    for _ in range(2):  # two calls in a row share the fixed scratch
        out = T.dense_attention_noalloc(Q, K, V)
        torch.cuda.synchronize()
        diff = (out.float() - ref.float()).abs()
        assert diff.max().item() <= max_tol and diff.mean().item() <= mean_tol
    assert ws.status() == T.TLSP_OK
    # both entry points run the same dense kernel, so also hold a few rows of
    # each head against the fp64 oracle's dense attention on the same inputs
    from oracle import oracle as orc
    rows = [0, n_q // 2, n_q - 1]
    for b in range(B):
        for h in range(H):
            Xq, Xk, Xv = (X[b, h].double().cpu().numpy() for X in (Q, K, V))
            O_ref, _ = orc.dense(Xq[rows], Xk, Xv)
            d_or = abs(out[b, h, rows].double().cpu().numpy() - O_ref)
            assert d_or.max() <= max_tol and d_or.mean() <= mean_tol, (b, h, d_or.max())


def test_noalloc_refuses_sizes_beyond_its_scratch(T):
    d = T.Dims(1, 64, 65537, 128, 128, T.TLSP_BF16)   # 64 * 65537 > 4194304 queries
    p = ctypes.c_void_p(0x10000)                      # never dereferenced: rejected on the host
    before = T.launch_count()
    assert T.lib().tlsp_dense_attention_noalloc(ctypes.byref(d), p, p, p, p, None) == \
        T.TLSP_ERR_UNSUPPORTED
    assert T.launch_count() == before
