"""Host-level sequences of RIB attention layers.

"Rank-Factorized Implicit Neural Bias" (gist.science English summary,
Technical Summary §2.C): the window size cycles within a block (e.g.
16 -> 32 -> 64), and the positional tokens depend only on the window geometry
(Chinese summary §2.A), so one Qp/Kp set per (MLP, window size) serves every
window, batch entry and layer that shares it.  This module runs such layer
sequences through the library's entry points with a geometry cache; it adds
no arithmetic of its own.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Sequence

import torch

from . import (PositionMLP, PositionMLPGrad, PosTokenCache, rib_window_attn_bwd,
               rib_window_attn_fwd)


@dataclass
class LayerSpec:
    window: int
    shift: int
    mlp: PositionMLP


@dataclass
class LayerState:
    out: torch.Tensor
    lse: torch.Tensor


class RIBLayerStack:
    """A sequence of RIB window-attention layers (a cyclic window schedule, or
    a stack of layers that alternate the shift) sharing one position-token
    cache."""

    def __init__(self, layers: Sequence[LayerSpec], cache: Optional[PosTokenCache] = None):
        self.layers = list(layers)
        self.cache = cache if cache is not None else PosTokenCache()

    def tokens(self, i: int):
        spec = self.layers[i]
        _, _, qp16, kp16 = self.cache.get(spec.mlp, spec.window)
        return qp16, kp16

    def forward(self, qkvs: Sequence[torch.Tensor]) -> List[LayerState]:
        """qkvs[i]: bf16 [B][H][W][3][heads][32] input of layer i."""
        states = []
        for i, (spec, qkv) in enumerate(zip(self.layers, qkvs)):
            qp16, kp16 = self.tokens(i)
            out, lse = rib_window_attn_fwd(qkv, spec.window, spec.shift, qp16, kp16,
                                           rank=spec.mlp.rank)
            states.append(LayerState(out, lse))
        return states

    def backward(self, qkvs: Sequence[torch.Tensor], states: Sequence[LayerState],
                 douts: Sequence[torch.Tensor], mlp_grads: bool = True):
        """Per-layer gradients (dqkv, dqp, dkp and, if requested, the MLP
        weight gradients) for upstream gradients douts[i]."""
        grads = []
        for i, (spec, qkv, st, dout) in enumerate(zip(self.layers, qkvs, states, douts)):
            qp16, kp16 = self.tokens(i)
            grads.append(rib_window_attn_bwd(qkv, st.out, dout, st.lse, spec.window, spec.shift,
                                             qp16, kp16, rank=spec.mlp.rank,
                                             mlp=spec.mlp if mlp_grads else None))
        return grads
