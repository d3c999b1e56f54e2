"""Seeded synthetic inputs for RIB windowed attention.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic, so both the fp64 oracle (tests, CPU baseline) and the
CUDA path can be fed from it without sharing any computation.

Workloads (the five shapes the benchmark and the parity tests run):

  tiny      B=1, 64x64 map, 16x16 windows, no shift, 3 heads, d=32, rank 16,
            MLP 64->64->48; features generated in fp32 and rounded to bf16
  w32       B=4, 128x128 map, 32x32 windows, shift 16, 6 heads, d=32,
            rank 16, MLP 64->128->96, fwd+bwd
  cyclic    B=8, 192x192 map, three layers with windows 16/32/64 and shifts
            0/16/0 (half a window on the middle layer), fwd+bwd
  w96train  B=4, 192x192 map, 96x96 windows, shift 48, fwd+bwd with MLP grads
  w96infer  B=1, 576x384 map, 96x96 windows, 12 layers with shifts 0,48,0,...,
            forward only, one MLP shared by every layer

Recipe: torch CPU generator, randn in fp32, then cast.  Features and upstream
gradients ~ N(0,1); MLP weights ~ N(0, 0.02), biases 0 (the benchmark recipe).
With those weights the bias logits are ~1e-4 and invisible, so parity tests
also use a "strong" variant: weights N(0, (1.5/sqrt(fan_in))^2), biases
N(0, 0.1^2), which gives Qp/Kp entries of std ~1 and bias logits of std
~0.65 (max ~6), the size of the content logits (std ~0.8 for N(0,1)
features, d=32).  Fourier frequencies default to pi*(k+1), k < 16.  Seed: 0 for tiny, the workload's index otherwise, plus
1000 per layer.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional

import torch

__all__ = [
    "Workload", "WORKLOADS", "get_workload", "default_freqs", "make_qkv",
    "make_dout", "make_mlp", "make_layer_inputs", "make_features", "make_cla", "ClaParams",
]


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    height: int
    width: int
    windows: tuple          # window side per layer
    shifts: tuple           # cyclic shift per layer
    heads: int = 6
    head_dim: int = 32
    rank: int = 16
    n_freq: int = 16
    hidden: int = 128
    seed: int = 0
    backward: bool = True
    mlp_grads: bool = True
    shared_mlp: bool = False     # one MLP for every layer (w96infer)
    fp32_features: bool = False  # features drawn in fp32, rounded to bf16

    @property
    def layers(self) -> int:
        return len(self.windows)

    def tokens(self) -> int:
        return self.batch * self.height * self.width

    def units(self, layer: int = 0) -> int:
        m = self.windows[layer]
        return self.batch * (self.height // m) * (self.width // m) * self.heads


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 64, 64, (16,), (0,), heads=3, hidden=64,
                     seed=0, fp32_features=True),
    "w32": Workload("w32", 4, 128, 128, (32,), (16,), seed=1),
    "cyclic": Workload("cyclic", 8, 192, 192, (16, 32, 64), (0, 16, 0), seed=2),
    "w96train": Workload("w96train", 4, 192, 192, (96,), (48,), seed=3),
    "w96infer": Workload("w96infer", 1, 576, 384, (96,) * 12,
                         tuple(0 if l % 2 == 0 else 48 for l in range(12)),
                         seed=4, backward=False, mlp_grads=False,
                         shared_mlp=True),
}


def get_workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return replace(w, **overrides) if overrides else w


def _gen(seed: int, tag: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 64 + int(tag))
    return g


_TAG_QKV, _TAG_DOUT, _TAG_MLPQ, _TAG_MLPK, _TAG_MISC = 1, 2, 3, 4, 5
_TAG_X, _TAG_CLA = 6, 7


def default_freqs(n_freq: int = 16) -> torch.Tensor:
    """Angular Fourier frequencies pi*(k+1), k < n_freq, as fp32."""
    return torch.tensor([math.pi * (k + 1) for k in range(n_freq)],
                        dtype=torch.float32)


def make_qkv(batch, height, width, heads, head_dim, seed, dtype=torch.bfloat16,
             std=1.0) -> torch.Tensor:
    """qkv features [B][H][W][3][heads][head_dim], N(0, std^2), then cast."""
    g = _gen(seed, _TAG_QKV)
    x = torch.randn((batch, height, width, 3, heads, head_dim), generator=g,
                    dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def make_dout(batch, height, width, heads, head_dim, seed,
              dtype=torch.bfloat16) -> torch.Tensor:
    """Upstream gradient of the attention output [B][H][W][heads][head_dim]."""
    g = _gen(seed, _TAG_DOUT)
    x = torch.randn((batch, height, width, heads, head_dim), generator=g,
                    dtype=torch.float32)
    return x.to(dtype)


@dataclass
class MLPParams:
    """Two-layer position MLP, PyTorch Linear layout (weight [out][in])."""
    w1: torch.Tensor
    b1: torch.Tensor
    w2: torch.Tensor
    b2: torch.Tensor


def make_mlp(n_freq, hidden, heads, rank, seed, which, strong=False):
    """Weights of the q (which=0) or k (which=1) position MLP, fp32.

    d_in = 4*n_freq, d_out = heads*rank.  Default: weights N(0, 0.02),
    biases 0.  strong=True: weights N(0, (1.5/sqrt(fan_in))^2), biases
    N(0, 0.1^2)."""
    g = _gen(seed, _TAG_MLPQ if which == 0 else _TAG_MLPK)
    d_in, d_out = 4 * n_freq, heads * rank
    s1 = 1.5 / math.sqrt(d_in) if strong else 0.02
    s2 = 1.5 / math.sqrt(hidden) if strong else 0.02
    w1 = torch.randn((hidden, d_in), generator=g) * s1
    w2 = torch.randn((d_out, hidden), generator=g) * s2
    if strong:
        b1 = torch.randn((hidden,), generator=g) * 0.1
        b2 = torch.randn((d_out,), generator=g) * 0.1
    else:
        b1 = torch.zeros(hidden)
        b2 = torch.zeros(d_out)
    return MLPParams(w1.float().contiguous(), b1.float().contiguous(),
                     w2.float().contiguous(), b2.float().contiguous())


def make_layer_inputs(w: Workload, layer: int = 0, strong: bool = False,
                      with_dout: Optional[bool] = None, qkv_dtype=torch.bfloat16):
    """All host-side inputs of one layer of workload w (CPU tensors).
    qkv_dtype=torch.float32 keeps the features unrounded (the fp32 path)."""
    seed = w.seed + 1000 * layer
    mlp_seed = w.seed if w.shared_mlp else seed
    qkv = make_qkv(w.batch, w.height, w.width, w.heads, w.head_dim, seed, dtype=qkv_dtype)
    out = {
        "qkv": qkv,
        "freqs": default_freqs(w.n_freq),
        "mlp_q": make_mlp(w.n_freq, w.hidden, w.heads, w.rank, mlp_seed, 0,
                          strong),
        "mlp_k": make_mlp(w.n_freq, w.hidden, w.heads, w.rank, mlp_seed, 1,
                          strong),
        "window": w.windows[layer],
        "shift": w.shifts[layer],
    }
    if with_dout if with_dout is not None else w.backward:
        out["dout"] = make_dout(w.batch, w.height, w.width, w.heads,
                                w.head_dim, seed)
    return out


def make_features(batch, height, width, channels, seed, dtype=torch.bfloat16):
    """Layer input feature map x [B][H][W][C] ~ N(0, 1), then cast (the
    input of the convolutional local attention gate)."""
    g = _gen(seed, _TAG_X)
    return torch.randn((batch, height, width, channels), generator=g,
                       dtype=torch.float32).to(dtype)


@dataclass
class ClaParams:
    """Convolutional local attention gate weights, fp32: depth-wise 3x3
    (w_dw [C][3][3], b_dw [C]) and point-wise 1x1 (w_pw [C][C], b_pw [C])."""
    w_dw: torch.Tensor
    b_dw: torch.Tensor
    w_pw: torch.Tensor
    b_pw: torch.Tensor


def make_cla(channels, seed):
    """CLA gate weights: w_dw ~ N(0, (1/3)^2) (a 3x3 tap sum of unit
    variance), w_pw ~ N(0, 1/C) (unit-variance pre-activation), biases
    N(0, 0.1^2), so the gate spans the sigmoid's whole range."""
    g = _gen(seed, _TAG_CLA)
    C = channels
    w_dw = torch.randn((C, 3, 3), generator=g) / 3.0
    b_dw = torch.randn((C,), generator=g) * 0.1
    w_pw = torch.randn((C, C), generator=g) / math.sqrt(C)
    b_pw = torch.randn((C,), generator=g) * 0.1
    return ClaParams(w_dw.contiguous(), b_dw.contiguous(), w_pw.contiguous(), b_pw.contiguous())


def randn(shape, seed, tag=_TAG_MISC, std=1.0, dtype=torch.float32):
    """Generic seeded N(0, std^2) draw for tests."""
    g = _gen(seed, tag)
    return (torch.randn(shape, generator=g, dtype=torch.float32) * std).to(dtype)
