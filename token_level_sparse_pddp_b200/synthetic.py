"""Seeded synthetic Q/K/V for the five workloads of the MC-Sparse hot path.

This module holds no arithmetic of the method itself (no attention, grouping or
selection). It only draws inputs; both the CUDA path and the fp64 oracle are fed
the same rounded tensors it returns.

Recipe (the pages evaluate on video diffusion transformers whose weights and
prompts are not available; these fields stand in for their attention inputs):

* Tokens lie on a (frames x height x width) grid and are flattened as
  n = (t * H + y) * W + x  (frame-major, the (f, h, w) layout of the video DiT
  token grid in "MonarchRT", section 3).
* For each of Q, K, V and each (batch, head) independently: 4 sinusoids with
  integer frequencies (f_t, f_y, f_x) drawn uniformly from {0, 1, 2, 3}, a
  per-channel amplitude a ~ N(0, 1) / 2 and phase phi ~ U[0, 2 pi);
  x[t, y, x, c] = sum_s a[s, c] * sin(2 pi (f_t t / T + f_y y / H + f_x x / W) + phi[s, c])
  plus N(0, 0.5^2) noise.
* The field is kept as an fp32 master copy and rounded to bf16 (round to
  nearest even) for the bf16 workloads.
* Before each step s >= 1 the master copies drift: master += drift * N(0, 1).
* The autoregressive-chunk workload draws its queries on frames 18..20 of the
  21-frame grid the keys and values live on.

Random numbers come from numpy's PCG64 generator, so the inputs are the same on
every machine for a given seed.
"""
from __future__ import annotations

import dataclasses
from typing import Iterator, Optional, Tuple

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "workload", "InputStream", "field"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    head_dim: int
    grid: Tuple[int, int, int]            # (T, H, W) of the key/value grid
    q_frames: Optional[Tuple[int, int]]   # [first, last] query frame; None = same grid as K/V
    dtype: str                            # "f32" or "bf16"
    group_size: int
    k: int
    schedule: str                         # 'A' = anchor step, 'R' = reuse step
    drift: float
    seed: int

    @property
    def n_kv(self) -> int:
        t, h, w = self.grid
        return t * h * w

    @property
    def n_q(self) -> int:
        t, h, w = self.grid
        if self.q_frames is None:
            return t * h * w
        return (self.q_frames[1] - self.q_frames[0] + 1) * h * w

    @property
    def num_groups(self) -> int:
        return -(-self.n_q // self.group_size)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def reuse_flops(self) -> float:
        """Executed tensor flops of one reuse step: QK^T and PV on the k selected tokens."""
        return 4.0 * self.batch * self.heads * self.n_q * self.k * self.head_dim

    def dense_flops(self) -> float:
        """Flops of one dense attention pass over all n_kv tokens."""
        return 4.0 * self.batch * self.heads * self.n_q * self.n_kv * self.head_dim


WORKLOADS = [
    Workload("tiny-fp32-N128", 1, 2, 64, (2, 8, 8), None, "f32", 16, 32, "AR", 0.05, 0),
    Workload("bf16-N1024", 1, 8, 128, (4, 16, 16), None, "bf16", 64, 256, "ARR", 0.03, 1),
    Workload("wan1.3b-N32760", 1, 12, 128, (21, 30, 52), None, "bf16", 128, 1664, "ARAR", 0.02, 2),
    Workload("ar-chunk-Nq4680-Nkv32760", 1, 12, 128, (21, 30, 52), (18, 20), "bf16", 128, 2048,
             "ARRR", 0.02, 3),
    Workload("large-dit-N75600", 1, 40, 128, (21, 45, 80), None, "bf16", 128, 7552, "ARRARR",
             0.015, 4),
]


def workload(i_or_name) -> Workload:
    if isinstance(i_or_name, int):
        return WORKLOADS[i_or_name]
    for w in WORKLOADS:
        if w.name == i_or_name:
            return w
    raise KeyError(i_or_name)


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=key)))


def field(rng: np.random.Generator, d: int, grid, frames) -> np.ndarray:
    """One fp32 field [N, d] of one head on the frames `frames` of `grid`.

    sin(a + phi) is expanded as sin(a) cos(phi) + cos(a) sin(phi) so the sum
    over sinusoids becomes a small matrix product.
    """
    T, H, W = grid
    t = np.asarray(frames, dtype=np.float64)[:, None, None]
    y = np.arange(H, dtype=np.float64)[None, :, None]
    x = np.arange(W, dtype=np.float64)[None, None, :]
    n = len(frames) * H * W
    freqs = rng.integers(0, 4, size=(4, 3))
    amp = rng.standard_normal((4, d)) / 2.0
    phase = rng.uniform(0.0, 2.0 * np.pi, size=(4, d))
    basis = np.empty((n, 8), dtype=np.float64)
    coef = np.empty((8, d), dtype=np.float64)
    for s in range(4):
        ft, fy, fx = freqs[s]
        ang = 2.0 * np.pi * (ft * t / T + fy * y / H + fx * x / W)
        ang = np.broadcast_to(ang, (len(frames), H, W)).reshape(n)
        basis[:, 2 * s] = np.sin(ang)
        basis[:, 2 * s + 1] = np.cos(ang)
        coef[2 * s] = amp[s] * np.cos(phase[s])
        coef[2 * s + 1] = amp[s] * np.sin(phase[s])
    noise = rng.standard_normal((n, d), dtype=np.float32) * np.float32(0.5)
    return (basis @ coef).astype(np.float32) + noise


def _round(master: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(master)
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    return t.clone()


class InputStream:
    """Yields (step, kind, Q, K, V) for a workload's schedule, drifting between steps.

    Q, K, V are CPU torch tensors [B, len(head_ids), N, d] in the workload dtype.
    Every (tensor, batch, head) field and every (tensor, batch, head, step)
    drift draws from its own generator spawned from the workload seed, so a
    stream restricted to some heads (`head_ids`) sees exactly the numbers the
    full stream holds for those heads. `batch_offset` shifts the batch index
    the generators are keyed on: a stream with batch_offset = r * B holds
    batch elements r*B .. r*B + B - 1 of a larger batch (one data-parallel
    shard of it).
    """

    def __init__(self, wl: Workload, head_ids=None, steps: Optional[int] = None,
                 batch_offset: int = 0):
        self.wl = wl
        self.head_ids = list(range(wl.heads)) if head_ids is None else list(head_ids)
        self.steps = len(wl.schedule) if steps is None else steps
        self.batch_offset = int(batch_offset)

    def __iter__(self) -> Iterator[Tuple[int, str, torch.Tensor, torch.Tensor, torch.Tensor]]:
        wl = self.wl
        T, H, W = wl.grid
        q_frames = list(range(T)) if wl.q_frames is None else list(
            range(wl.q_frames[0], wl.q_frames[1] + 1))
        kv_frames = list(range(T))
        nh = len(self.head_ids)
        b0 = self.batch_offset
        masters = []
        for which, frames in enumerate((q_frames, kv_frames, kv_frames)):
            n = len(frames) * H * W
            m = np.empty((wl.batch, nh, n, wl.head_dim), dtype=np.float32)
            for b in range(wl.batch):
                for j, h in enumerate(self.head_ids):
                    m[b, j] = field(_rng(wl.seed, which, b0 + b, h), wl.head_dim, wl.grid,
                                    frames)
            masters.append(m)
        for s in range(self.steps):
            if s > 0:
                for which, m in enumerate(masters):
                    for b in range(wl.batch):
                        for j, h in enumerate(self.head_ids):
                            g = _rng(wl.seed, which, b0 + b, h, s)
                            m[b, j] += np.float32(wl.drift) * g.standard_normal(
                                m.shape[2:], dtype=np.float32)
            kind = wl.schedule[s % len(wl.schedule)]
            yield (s, kind, *(_round(m, wl.dtype) for m in masters))
