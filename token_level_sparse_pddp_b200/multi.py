"""Data-parallel sharding of the hot path over ranks (one process per GPU).

Every (batch, head) problem of the path is independent: PDDP grouping, the
exact group scores, the top-k selection and both sparse passes are defined
per head (MC-Sparse review, section 3: groups, scores and the cached
selection belong to one head's attention). A job of `world * B` batch
elements therefore gives rank r the elements [r*B, (r+1)*B) and runs them
with no exchange of data between ranks (weak scaling); alternatively the
heads of a fixed batch are split over the ranks (`head_shard`, strong
scaling). The only collectives are the ones a
measurement needs: a barrier around the timed region and a max over ranks of
the measured times.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass
from typing import List, Sequence

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local_rank: int

    @property
    def is_root(self) -> bool:
        return self.rank == 0


def rank_info() -> RankInfo:
    """Rank, world size and local rank from the launcher's environment
    (torchrun sets RANK / WORLD_SIZE / LOCAL_RANK; a plain run is rank 0 of 1)."""
    return RankInfo(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def batch_offset(batch_per_rank: int, rank: int) -> int:
    """First global batch index held by `rank` when every rank holds
    `batch_per_rank` consecutive elements."""
    if batch_per_rank < 1 or rank < 0:
        raise ValueError("batch_per_rank >= 1 and rank >= 0 required")
    return rank * batch_per_rank


def shard_bounds(global_batch: int, world: int, rank: int) -> range:
    """Global batch indices of `rank` (equal shards; global_batch must divide)."""
    if world < 1 or not 0 <= rank < world or global_batch % world:
        raise ValueError(f"cannot shard a batch of {global_batch} over {world} ranks")
    per = global_batch // world
    return range(batch_offset(per, rank), batch_offset(per, rank) + per)


def head_shard(heads: int, world: int, rank: int) -> range:
    """Heads of `rank` when one batch element's heads are split over the ranks
    (contiguous, as equal as possible: the first heads % world ranks hold one
    more). Grouping, scores, selection and both sparse passes are per head, so
    the shards need no exchange either; this splits a fixed problem (strong
    scaling) where batch sharding grows it (weak scaling)."""
    if world < 1 or not 0 <= rank < world or heads < world:
        raise ValueError(f"cannot split {heads} heads over {world} ranks")
    base, extra = divmod(heads, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def init(info: RankInfo, backend: str, device=None, timeout_s: float = 120.0) -> None:
    """Joins the process group when world > 1 (short timeout: ranks that wait
    on a missing peer end with an error instead of hanging)."""
    if info.world <= 1:
        return
    kw = {}
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, rank=info.rank, world_size=info.world,
                            timeout=datetime.timedelta(seconds=timeout_s), **kw)


def barrier(info: RankInfo) -> None:
    if info.world > 1:
        dist.barrier()


def max_over_ranks(info: RankInfo, values: Sequence[float], device=None) -> List[float]:
    """Element-wise max of `values` over all ranks (identity on one rank)."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if info.world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu().tolist()]


def aggregate_rate(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Whole-job rate: the units all ranks processed over the slowest rank's time."""
    if seconds_max <= 0:
        raise ValueError("non-positive time")
    return units_per_rank * world / seconds_max


def finish(info: RankInfo) -> None:
    if info.world > 1 and dist.is_initialized():
        dist.destroy_process_group()
