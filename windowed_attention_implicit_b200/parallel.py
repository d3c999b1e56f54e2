"""Data-parallel plumbing for RIB window attention training.

Every (batch, window, head) unit is an independent attention problem, so the
forward needs no communication: ranks split the batch.  The one exchange is
in the backward: the position-MLP weight gradients are sums over every
window of every batch entry, so the per-rank partial sums are all-reduced
(sum) once per step -- one flat fp32 buffer, one collective (NCCL on GPUs,
gloo on CPU).
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import torch
import torch.distributed as dist

from . import PositionMLP, PositionMLPGrad


def shard_batch(global_batch: int, world: int, rank: int) -> slice:
    """Contiguous batch slice of `rank`; the first (global_batch % world)
    ranks take one extra entry."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


class FlatGrads:
    """Position-MLP gradients as views of one contiguous fp32 buffer, so the
    cross-rank sum is a single all-reduce."""

    ORDER = ("q_dw1", "q_db1", "q_dw2", "q_db2", "k_dw1", "k_db1", "k_dw2", "k_db2")

    def __init__(self, shapes: Sequence[Tuple[int, ...]], device, dtype=torch.float32):
        sizes = [int(torch.Size(s).numel()) for s in shapes]
        self.flat = torch.zeros(sum(sizes), device=device, dtype=dtype)
        self.views: List[torch.Tensor] = []
        off = 0
        for s, n in zip(shapes, sizes):
            self.views.append(self.flat[off:off + n].view(s))
            off += n

    @classmethod
    def for_mlp(cls, mlp: PositionMLP) -> "FlatGrads":
        shapes = [tuple(t.shape) for t in (mlp.q_w1, mlp.q_b1, mlp.q_w2, mlp.q_b2,
                                           mlp.k_w1, mlp.k_b1, mlp.k_w2, mlp.k_b2)]
        return cls(shapes, mlp.q_w1.device)

    def as_grad(self) -> PositionMLPGrad:
        return PositionMLPGrad(*self.views)

    def named(self):
        return dict(zip(self.ORDER, self.views))


def allreduce_grads(flat: torch.Tensor, group=None) -> torch.Tensor:
    """Sums `flat` over the ranks of `group` in place (no-op on one rank)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    return flat
