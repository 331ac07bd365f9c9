"""Data-parallel sharding over ranks, on CPU with the gloo backend (world 2).

The path has no exchange step: each rank runs its own batch elements. These
tests check that the shards of a global batch hold exactly the inputs the
unsharded stream holds for those elements, that the per-rank results (oracle
PDDP grouping, anchor step and reuse step per head) equal the unsharded
results, and that the measurement collectives (max over ranks, barrier) and the
whole-job rate behave as the benchmark uses them.
"""
import dataclasses
import os
import pickle
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from oracle import oracle as orc  # noqa: E402
from token_level_sparse_pddp_b200 import multi  # noqa: E402
from token_level_sparse_pddp_b200.synthetic import InputStream, workload  # noqa: E402

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _path_results(wl, stream):
    """Oracle results of one anchor period for every (batch, head) of a stream."""
    it = iter(stream)
    _, _, Qa, Ka, Va = next(it)
    _, _, Qr, Kr, Vr = next(it)
    gs, k = wl.group_size, wl.k
    out = {}
    for b in range(Qa.shape[0]):
        for h in range(Qa.shape[1]):
            groups = orc.pddp(Qa[b, h].double().numpy(), gs)
            anc = orc.anchor_groups(Qa[b, h], Ka[b, h], Va[b, h], groups, gs, k)
            reu = orc.reuse_groups(Qr[b, h], Kr[b, h], Vr[b, h], groups, gs,
                                   {g: a["idx"] for g, a in anc.items()},
                                   {g: a["R"] for g, a in anc.items()})
            out[(b, h)] = dict(groups=groups, idx=np.stack([anc[g]["idx"] for g in sorted(anc)]),
                               R=np.concatenate([anc[g]["R"] for g in sorted(anc)]),
                               O=np.concatenate([reu[g] for g in sorted(reu)]),
                               Q=Qa[b, h].numpy().copy())
    return out


def _path_results_heads(wl, head_ids):
    """As _path_results, for the given heads of batch element 0 (keys: head ids)."""
    res = _path_results(wl, InputStream(wl, head_ids=head_ids, steps=2))
    return {head_ids[h]: v for (b, h), v in res.items()}


def _worker_heads(rank, port, out_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank))
    info = multi.rank_info()
    multi.init(info, "gloo", timeout_s=60)
    wl = dataclasses.replace(workload(0), heads=3)  # uneven: 2 heads on rank 0, 1 on rank 1
    mine = list(multi.head_shard(wl.heads, info.world, info.rank))
    res = _path_results_heads(wl, mine)
    gathered = [None] * info.world
    dist.all_gather_object(gathered, res)
    multi.barrier(info)
    if info.is_root:
        with open(out_path, "wb") as f:
            pickle.dump(gathered, f)
    multi.finish(info)


def _worker(rank, port, out_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank))
    info = multi.rank_info()
    multi.init(info, "gloo", timeout_s=60)
    wl = workload(0)
    res = _path_results(wl, InputStream(wl, steps=2,
                                        batch_offset=multi.batch_offset(wl.batch, info.rank)))
    gathered = [None] * info.world
    dist.all_gather_object(gathered, res)
    mx = multi.max_over_ranks(info, [float(rank + 1), -float(rank), 0.5])
    multi.barrier(info)
    if info.is_root:
        with open(out_path, "wb") as f:
            pickle.dump(dict(gathered=gathered, mx=mx, world=info.world), f)
    multi.finish(info)


@pytest.fixture(scope="module")
def sharded(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("gloo") / "res.pkl")
    mp.start_processes(_worker, args=(_free_port(), out), nprocs=WORLD, join=True,
                       start_method="spawn")
    with open(out, "rb") as f:
        return pickle.load(f)


def test_max_over_ranks(sharded):
    assert sharded["world"] == WORLD
    assert sharded["mx"] == [float(WORLD), 0.0, 0.5]


def test_shards_equal_slices_of_global_batch(sharded):
    wl = workload(0)
    glob = dataclasses.replace(wl, batch=WORLD * wl.batch)
    ref = _path_results(glob, InputStream(glob, steps=2))
    for r, res in enumerate(sharded["gathered"]):
        for (b, h), v in res.items():
            g = ref[(multi.batch_offset(wl.batch, r) + b, h)]
            assert np.array_equal(v["Q"], g["Q"])
            assert np.array_equal(v["groups"], g["groups"])
            assert np.array_equal(v["idx"], g["idx"])
            assert np.array_equal(v["R"], g["R"])
            assert np.array_equal(v["O"], g["O"])
    # the two shards are different data
    a, b = (sharded["gathered"][r][(0, 0)]["Q"] for r in range(WORLD))
    assert not np.array_equal(a, b)


def test_shard_bounds_and_rate():
    assert list(multi.shard_bounds(8, 4, 2)) == [4, 5]
    assert [list(multi.shard_bounds(6, 2, r)) for r in range(2)] == [[0, 1, 2], [3, 4, 5]]
    with pytest.raises(ValueError):
        multi.shard_bounds(5, 2, 0)
    with pytest.raises(ValueError):
        multi.shard_bounds(4, 2, 2)
    assert multi.aggregate_rate(10.0, 4, 2.0) == 20.0
    with pytest.raises(ValueError):
        multi.aggregate_rate(1.0, 1, 0.0)


def test_single_rank_is_identity():
    info = multi.RankInfo(0, 1, 0)
    multi.init(info, "gloo")  # no process group for one rank
    assert not dist.is_initialized()
    assert multi.max_over_ranks(info, [3.0, -1.0]) == [3.0, -1.0]
    multi.barrier(info)
    multi.finish(info)


def _bench_reference(rank: int):
    import subprocess
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank),
               OMP_NUM_THREADS="2")
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--workload", "0", "--steps", "1", "--warmup", "0", "--gpus", "2"],
                          env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_only_on_rank0():
    import json
    r1 = _bench_reference(1)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _bench_reference(0)
    assert r0.returncode == 0, r0.stderr
    lines = [l for l in r0.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0



def test_head_shard_bounds():
    assert [list(multi.head_shard(12, 5, r)) for r in range(5)] == \
        [[0, 1, 2], [3, 4, 5], [6, 7], [8, 9], [10, 11]]
    assert list(multi.head_shard(40, 8, 7)) == list(range(35, 40))
    for heads, world in ((12, 8), (40, 8), (3, 2), (7, 7)):
        got = [h for r in range(world) for h in multi.head_shard(heads, world, r)]
        assert got == list(range(heads))
    with pytest.raises(ValueError):
        multi.head_shard(3, 4, 0)
    with pytest.raises(ValueError):
        multi.head_shard(8, 2, 2)


def test_head_shards_equal_unsharded_heads(tmp_path):
    """Heads split over two gloo ranks: every head's grouping, selection, residual and
    reuse output equal the unsharded run's for that head."""
    out = str(tmp_path / "heads.pkl")
    mp.start_processes(_worker_heads, args=(_free_port(), out), nprocs=WORLD, join=True,
                       start_method="spawn")
    with open(out, "rb") as f:
        gathered = pickle.load(f)
    wl = dataclasses.replace(workload(0), heads=3)
    ref = _path_results_heads(wl, list(range(wl.heads)))
    seen = {}
    for res in gathered:
        seen.update(res)
    assert sorted(seen) == list(range(wl.heads))
    for h, v in seen.items():
        for key in ("Q", "groups", "idx", "R", "O"):
            assert np.array_equal(v[key], ref[h][key]), (h, key)
