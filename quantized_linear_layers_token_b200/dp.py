"""Data-parallel exchange of the targeted-momentum statistics.

Quaff notes, 目标动量缩放: beta_i is built from max_m |X[m, O_i]| over the
step's tokens.  When the tokens of a step are sharded over ranks, every rank
computes the column maxima of its own shard (qlin_outlier_colmax) and one
all-reduce(MAX) of all layers' maxima, packed into one vector, gives every
rank the global maxima; each rank then applies the recurrence itself
(qlin_momentum_update), so all replicas keep the same state s.  The maximum
is exact and order-free, so the result is bit-identical to the update over
the unsharded batch.
"""
from __future__ import annotations

from typing import Sequence

import torch


class ColmaxExchange:
    """One flat fp32 buffer holding the outlier column maxima of several
    layers (layer j at [offset[j], offset[j] + n_outlier[j])), reduced with a
    single all-reduce(MAX) per step."""

    def __init__(self, n_outliers: Sequence[int], device: torch.device | str = "cpu"):
        self.n_outliers = [int(n) for n in n_outliers]
        if any(n < 0 for n in self.n_outliers):
            raise ValueError("negative outlier count")
        self.offsets = []
        total = 0
        for n in self.n_outliers:
            self.offsets.append(total)
            total += n
        self.total = total
        # at least one element so the collective always has a buffer
        self.buf = torch.zeros(max(total, 1), dtype=torch.float32, device=device)

    def view(self, j: int) -> torch.Tensor:
        """The slice that layer j's column maxima are written into."""
        o = self.offsets[j]
        return self.buf[o:o + self.n_outliers[j]]

    def allreduce(self, group=None) -> None:
        """Combine every rank's maxima (collective: all ranks call it in the
        same order each step)."""
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
            dist.all_reduce(self.buf, op=dist.ReduceOp.MAX, group=group)
