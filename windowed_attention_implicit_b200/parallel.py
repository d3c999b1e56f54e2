"""Data-parallel plumbing for RIB window attention training.

Every (batch, window, head) unit is an independent attention problem, so the
forward needs no communication: ranks split the batch.  The one exchange is
in the backward: the position-MLP weight gradients are sums over every
window of every batch entry, so the per-rank partial sums are all-reduced
(sum) once per step -- one flat fp32 buffer, one collective (NCCL on GPUs,
gloo on CPU).  With the convolutional local attention gate in the step, its
four weight gradients (sums over every pixel) join the same buffer.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

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
    """Gradients as views of one contiguous buffer, so that the cross-rank
    sum is a single all-reduce.  Layouts: the position MLPs (`for_mlp`), the
    CLA gate (`for_cla`), or both (`for_mlp_and_cla`, MLP first)."""

    ORDER = ("q_dw1", "q_db1", "q_dw2", "q_db2", "k_dw1", "k_db1", "k_dw2", "k_db2")
    CLA_ORDER = ("cla_dw_dw", "cla_db_dw", "cla_dw_pw", "cla_db_pw")

    def __init__(self, shapes: Sequence[Tuple[int, ...]], device, dtype=torch.float32,
                 names: Optional[Sequence[str]] = None):
        if names is None:
            names = self.ORDER if len(shapes) == len(self.ORDER) else \
                tuple(f"g{i}" for i in range(len(shapes)))
        if len(names) != len(shapes):
            raise ValueError("one name per gradient shape")
        self.names = tuple(names)
        sizes = [int(torch.Size(s).numel()) for s in shapes]
        self.flat = torch.zeros(sum(sizes), device=device, dtype=dtype)
        self.views: List[torch.Tensor] = []
        off = 0
        for s, n in zip(shapes, sizes):
            self.views.append(self.flat[off:off + n].view(s))
            off += n

    @staticmethod
    def _mlp_shapes(mlp: PositionMLP):
        return [tuple(t.shape) for t in (mlp.q_w1, mlp.q_b1, mlp.q_w2, mlp.q_b2,
                                         mlp.k_w1, mlp.k_b1, mlp.k_w2, mlp.k_b2)]

    @staticmethod
    def _cla_shapes(channels: int):
        C = int(channels)
        if C <= 0:
            raise ValueError("channels must be positive")
        return [(C, 3, 3), (C,), (C, C), (C,)]

    @classmethod
    def for_mlp(cls, mlp: PositionMLP) -> "FlatGrads":
        return cls(cls._mlp_shapes(mlp), mlp.q_w1.device, names=cls.ORDER)

    @classmethod
    def for_cla(cls, channels: int, device) -> "FlatGrads":
        """dW_dw [C][3][3], db_dw [C], dW_pw [C][C], db_pw [C]."""
        return cls(cls._cla_shapes(channels), device, names=cls.CLA_ORDER)

    @classmethod
    def for_mlp_and_cla(cls, mlp: PositionMLP, channels: int) -> "FlatGrads":
        return cls(cls._mlp_shapes(mlp) + cls._cla_shapes(channels), mlp.q_w1.device,
                   names=cls.ORDER + cls.CLA_ORDER)

    def as_grad(self) -> PositionMLPGrad:
        """The position-MLP views as the binding's gradient record."""
        if self.names[:len(self.ORDER)] != self.ORDER:
            raise ValueError("this buffer holds no position-MLP gradients")
        return PositionMLPGrad(*self.views[:len(self.ORDER)])

    def cla(self) -> Dict[str, torch.Tensor]:
        """The CLA views under the keys rib_cla_bwd returns (dw_dw, db_dw,
        dw_pw, db_pw); copy that call's results into them before the sum."""
        got = {n[len("cla_"):]: v for n, v in zip(self.names, self.views) if n.startswith("cla_")}
        if len(got) != len(self.CLA_ORDER):
            raise ValueError("this buffer holds no CLA gradients")
        return got

    def named(self):
        return dict(zip(self.names, self.views))


def allreduce_grads(flat: torch.Tensor, group=None) -> torch.Tensor:
    """Sums `flat` over the ranks of `group` in place (no-op on one rank)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    return flat
