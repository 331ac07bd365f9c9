"""The C-ABI library loads, exports every symbol include/tlsp.h declares, and
validates arguments on the host (no kernel is launched by these tests)."""
import ctypes
import os
import re
import subprocess

import pytest

from token_level_sparse_pddp_b200 import build as tlsp_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tlsp.h")


@pytest.fixture(scope="module")
def T():
    tlsp_build.build()
    from token_level_sparse_pddp_b200 import tlsp
    tlsp.lib()
    return tlsp


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tlsp_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("tlsp_group_queries", "tlsp_anchor_attention", "tlsp_reuse_attention",
                 "tlsp_topk_from_scores", "tlsp_split_from_projections",
                 "tlsp_group_queries_trace", "tlsp_get_device_status", "tlsp_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol(T):
    out = subprocess.run(["nm", "-D", "--defined-only", T.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (tlsp_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(T.lib(), n)
    assert sorted(T.EXPORTED) == declared_functions()


def test_group_counts(T):
    assert T.num_groups(128, 16) == 8
    assert T.num_groups(32760, 128) == 256
    assert T.num_groups(4680, 128) == 37
    assert T.num_groups(75600, 128) == 591
    assert T.num_groups(0, 16) == -1 and T.num_groups(5, 0) == -1
    assert [T.num_levels(n, 1) for n in (1, 2, 3, 4, 5)] == [0, 1, 2, 2, 3]
    assert T.num_levels(32760, 128) == 8 and T.num_levels(75600, 128) == 10


def test_workspace_bytes(T):
    d = T.Dims(1, 12, 32760, 32760, 128, T.TLSP_BF16)
    n = T.lib().tlsp_workspace_bytes(ctypes.byref(d), 128, 1664)
    # holds one batch of fp32 score rows (4 waves of 148 rows at n_kv = 32760),
    # not the whole [B, H, G, n_kv] matrix
    assert 592 * 32760 * 4 <= n < 12 * 256 * 32760 * 4
    d4 = T.Dims(1, 40, 75600, 75600, 128, T.TLSP_BF16)
    n4 = T.lib().tlsp_workspace_bytes(ctypes.byref(d4), 128, 7552)
    assert 296 * 75600 * 4 <= n4 < 1 << 30
    assert T.lib().tlsp_workspace_bytes(ctypes.byref(d), 128, 32761) == 0   # k > n_kv
    bad = T.Dims(1, 12, 32760, 32760, 96, T.TLSP_BF16)
    assert T.lib().tlsp_workspace_bytes(ctypes.byref(bad), 128, 1) == 0     # head_dim
    assert T.lib().tlsp_workspace_bytes(None, 128, 1) == 0


def test_status_strings(T):
    assert T.status_string(0) == "TLSP_OK"
    assert T.status_string(-5) == "TLSP_ERR_TIMEOUT"
    assert T.status_string(-6) == "TLSP_ERR_DEVICE_ASSERT"
    assert T.status_string(12345) == "TLSP_UNKNOWN_STATUS"


def test_validation_rejects_before_launch(T):
    L = T.lib()
    before = L.tlsp_launch_count()
    p = ctypes.c_void_p(0x10000)      # never dereferenced: every call below fails validation
    odd = ctypes.c_void_p(0x10004)    # not 16-byte aligned
    d = T.Dims(1, 2, 128, 128, 64, T.TLSP_F32)
    big = 1 << 40
    E_ARG, E_WS = T.TLSP_ERR_INVALID_ARG, T.TLSP_ERR_WORKSPACE
    # null / misaligned pointers
    assert L.tlsp_group_queries(ctypes.byref(d), None, 16, p, p, big, None) == E_ARG
    assert L.tlsp_group_queries(ctypes.byref(d), odd, 16, p, p, big, None) == E_ARG
    # bad shapes
    for bad in (T.Dims(0, 2, 128, 128, 64, 0), T.Dims(1, 2, 128, 128, 80, 0),
                T.Dims(1, 2, 0, 128, 64, 0), T.Dims(1, 2, 128, 128, 64, 7)):
        assert L.tlsp_group_queries(ctypes.byref(bad), p, 16, p, p, big, None) == E_ARG
    assert L.tlsp_group_queries(ctypes.byref(d), p, 0, p, p, big, None) == E_ARG
    # workspace too small
    assert L.tlsp_group_queries(ctypes.byref(d), p, 16, p, p, 64, None) == E_WS
    # k out of range
    assert L.tlsp_anchor_attention(ctypes.byref(d), p, p, p, p, 16, 129, p, p, p, None, p, big,
                                   None) == E_ARG
    assert L.tlsp_anchor_attention(ctypes.byref(d), p, p, p, p, 16, 0, p, p, p, None, p, big,
                                   None) == E_ARG
    assert L.tlsp_reuse_attention(ctypes.byref(d), p, p, p, p, 16, 32, p, None, p, p, big,
                                  None) == E_ARG
    assert L.tlsp_reuse_attention(ctypes.byref(d), p, p, odd, p, 16, 32, p, p, p, p, big,
                                  None) == E_ARG
    # the reuse step needs only the 256-byte status word
    assert L.tlsp_reuse_attention(ctypes.byref(d), p, p, p, p, 16, 32, p, p, p, p, 255,
                                  None) == E_WS
    assert L.tlsp_reuse_attention(ctypes.byref(d), p, p, p, p, 16, 32, p, p, p, None, 256,
                                  None) == E_ARG
    assert L.tlsp_topk_from_scores(p, 4, 10, 11, p, None, 0, None) == E_ARG
    assert L.tlsp_split_from_projections(p, p, 8, 9, p, p, None, 0, None) == E_ARG
    assert L.tlsp_debug_bounded_wait(None, 0, 10, None) == E_ARG
    # ablation calls
    E_UNS = T.TLSP_ERR_UNSUPPORTED
    assert L.tlsp_group_raster(ctypes.byref(d), 16, None, None) == E_ARG
    assert L.tlsp_group_raster(ctypes.byref(d), 0, p, None) == E_ARG
    assert L.tlsp_block_topk_from_scores(p, 4, 128, 129, 4, p, None, None) == E_ARG
    assert L.tlsp_block_topk_from_scores(p, 4, 128, 32, 0, p, None, None) == E_ARG
    assert L.tlsp_block_topk_from_scores(p, 4, 128, 32, 5, p, None, None) == E_UNS  # 5 ∤ 128
    assert L.tlsp_block_topk_from_scores(p, 4, 128, 30, 4, p, None, None) == E_UNS  # 4 ∤ 30
    assert L.tlsp_pooled_block_select(ctypes.byref(d), p, p, p, 16, 32, 5, p, None, p, big,
                                      None) == E_UNS
    assert L.tlsp_pooled_block_select(ctypes.byref(d), p, p, None, 16, 32, 4, p, None, p, big,
                                      None) == E_ARG
    assert L.tlsp_pooled_block_select(ctypes.byref(d), p, p, p, 16, 32, 4, p, None, p, 64,
                                      None) == E_WS
    assert L.tlsp_launch_count() == before
