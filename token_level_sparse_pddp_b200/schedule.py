"""The anchor / reuse schedule of MC-Sparse as a callable attention module.

MC-Sparse review, section 3: on an anchor denoising step the queries are grouped
(PDDP), dense attention runs, the exact per-group KV selection is taken and the
dense-sparse residual R = O_full - O_sparse is stored; on the reuse steps that
follow, only sparse attention over the cached selection runs and R is added
back. This module keeps that state (groups, selection, R, workspace) between
calls and decides, per step, which of the two the library runs. Everything it
computes goes through the C ABI; it holds no arithmetic of its own.

    attn = MCSparseAttention(group_size=128, k=1664, anchor_every=2)
    for step in range(num_steps):
        O = attn(Q[step], K[step], V[step])      # [B, H, n_q, d], input dtype
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import tlsp


class MCSparseAttention:
    """Stateful anchor / reuse attention over a sequence of denoising steps.

    Step s is an anchor step when `schedule` is given and schedule[s % len] is
    'A', else when s % anchor_every == 0 (so step 0 is always an anchor). A
    change of shape, dtype or device forces an anchor step.
    """

    def __init__(self, group_size: int, k: int, anchor_every: int = 2,
                 schedule: Optional[Sequence[str]] = None):
        if group_size < 1 or k < 1 or anchor_every < 1:
            raise ValueError("group_size, k and anchor_every must be >= 1")
        if schedule is not None and (not schedule or any(c not in "AR" for c in schedule)):
            raise ValueError("schedule must be a non-empty string of 'A' and 'R'")
        self.group_size, self.k, self.anchor_every = group_size, k, anchor_every
        self.schedule = None if schedule is None else "".join(schedule)
        self.step = 0
        self._key = None
        self.ws: Optional[tlsp.Workspace] = None
        self.groups = self.indices = self.R = None

    def is_anchor(self, step: int) -> bool:
        if self.schedule is not None:
            return self.schedule[step % len(self.schedule)] == "A"
        return step % self.anchor_every == 0

    def reset(self):
        """Forget the cached state; the next call is an anchor step."""
        self._key = None
        self.groups = self.indices = self.R = None
        self.step = 0

    def __call__(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor) -> torch.Tensor:
        key = (tuple(Q.shape), tuple(K.shape), Q.dtype, Q.device)
        anchor = self.is_anchor(self.step) or key != self._key
        if key != self._key:
            self.ws = tlsp.Workspace(tlsp.dims_of(Q, K), self.group_size, self.k,
                                     device=Q.device)
            self._key = key
        if anchor:
            self.groups = tlsp.group_queries(Q, self.group_size, self.ws)
            O, self.indices, self.R = tlsp.anchor_attention(Q, K, V, self.groups,
                                                            self.group_size, self.k, self.ws)
        else:
            O = tlsp.reuse_attention(Q, K, V, self.groups, self.group_size, self.k,
                                     self.indices, self.R, self.ws)
        self.last_was_anchor = anchor
        self.step += 1
        return O

    def status(self) -> int:
        """Device status of the workspace (after the caller's stream has finished)."""
        return self.ws.status() if self.ws is not None else tlsp.TLSP_OK
