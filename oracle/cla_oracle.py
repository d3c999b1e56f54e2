"""Plain fp64 CPU oracle of the convolutional local attention gate (CLA)
(TEST INFRASTRUCTURE ONLY: tests, the package smoke check and the
benchmark's CPU-baseline leg may use it; the CUDA library never does).

"Rank-Factorized Implicit Neural Bias" pages, convolutional local attention:
  [EN] gist.science English summary, Technical Summary §2.B: a lightweight
       convolutional path (depth-wise conv + point-wise conv + sigmoid)
       produces a gating map that modulates the self-attention output;
  [DE] gist.science/de, Methodik §B: the gating map G modulates the output,
       O' = O (element-wise) G;
  [ZH] gist.science/zh, §2.B: the depth-wise convolution is 3x3 and the
       point-wise one 1x1.

Readings where the pages are silent (each an argument or a documented
default, so tests can vary it):
  1. the convolutional path reads the layer's input feature map x with
     C = heads * d channels, laid out [B][H][W][C], so G has the shape of the
     attention output O viewed as [B][H][W][C] (channel = head * d + e);
  2. both convolutions carry a bias and nothing sits between them;
  3. the 3x3 depth-wise convolution is a cross-correlation with zero padding
     of one pixel on every side (output size = input size):
       y[b,i,j,c] = b_dw[c] + sum_{u,v in {0,1,2}} w_dw[c,u,v] x[b,i+u-1,j+v-1,c];
  4. the point-wise convolution is z[b,i,j,o] = b_pw[o] + sum_c w_pw[o,c] y[b,i,j,c],
     G = 1 / (1 + exp(-z));
  5. the gate acts on the full map (no windows, no shift): O' = O * G.

Pins (tests/test_cla_oracle.py): the convolutions against torch's fp64
conv2d, the sigmoid against its closed form, the backward against central
finite differences, plus the special cases w_pw = 0 (G = sigmoid(b_pw)
everywhere) and a single interior impulse.
"""
from __future__ import annotations

import numpy as np

__all__ = ["dw_conv3x3", "pw_conv", "sigmoid", "cla_gate", "cla_apply", "cla_backward"]


def _f64(a):
    if hasattr(a, "detach"):
        a = a.detach().cpu()
        if str(a.dtype) in ("torch.bfloat16", "torch.float16"):
            a = a.float()
        a = a.numpy()
    return np.asarray(a, dtype=np.float64)


def dw_conv3x3(x, w_dw, b_dw):
    """Reading 3: depth-wise 3x3 cross-correlation, zero padding 1.
    x [B][H][W][C], w_dw [C][3][3], b_dw [C] -> y [B][H][W][C]."""
    x = _f64(x)
    w = _f64(w_dw)
    B, H, W, C = x.shape
    xp = np.zeros((B, H + 2, W + 2, C))
    xp[:, 1:H + 1, 1:W + 1, :] = x
    y = np.broadcast_to(_f64(b_dw), (B, H, W, C)).copy()
    for u in range(3):
        for v in range(3):
            y += w[:, u, v] * xp[:, u:u + H, v:v + W, :]
    return y


def pw_conv(y, w_pw, b_pw):
    """Reading 4: point-wise convolution, z = y w_pw^T + b_pw per pixel.
    w_pw [C_out][C_in] (a 1x1 convolution's weight without its unit axes)."""
    return _f64(y) @ _f64(w_pw).T + _f64(b_pw)


def sigmoid(z):
    z = _f64(z)
    return 1.0 / (1.0 + np.exp(-z))


def cla_gate(x, w_dw, b_dw, w_pw, b_pw):
    """G = sigmoid(PW(DW3x3(x))): the CLA gating map ([EN] §2.B, [ZH] §2.B)."""
    return sigmoid(pw_conv(dw_conv3x3(x, w_dw, b_dw), w_pw, b_pw))


def cla_apply(o, g):
    """O' = O * G ([DE] §B); o [B][H][W][heads][d] or [B][H][W][C]."""
    o = _f64(o)
    return o * _f64(g).reshape(o.shape)


def cla_backward(x, w_dw, b_dw, w_pw, b_pw, o, d_out):
    """Gradients of L = sum(O' * dO') with O' = O * G(x).

    Returns dict with d_o (= dO' * G, the upstream gradient the attention
    backward receives), dx, dw_dw, db_dw, dw_pw, db_pw, all fp64; o and d_out
    are [B][H][W][C] (or any shape with that many elements)."""
    x = _f64(x)
    B, H, W, C = x.shape
    y = dw_conv3x3(x, w_dw, b_dw)
    g = sigmoid(pw_conv(y, w_pw, b_pw))
    o = _f64(o).reshape(B, H, W, C)
    dout = _f64(d_out).reshape(B, H, W, C)
    d_o = dout * g
    dz = dout * o * g * (1.0 - g)
    wpw = _f64(w_pw)
    dy = dz @ wpw
    dw_pw = np.einsum("bijo,bijc->oc", dz, y)
    db_pw = dz.sum(axis=(0, 1, 2))
    db_dw = dy.sum(axis=(0, 1, 2))
    wdw = _f64(w_dw)
    xp = np.zeros((B, H + 2, W + 2, C))
    xp[:, 1:H + 1, 1:W + 1, :] = x
    dxp = np.zeros_like(xp)
    dw_dw = np.zeros((C, 3, 3))
    for u in range(3):
        for v in range(3):
            dw_dw[:, u, v] = (dy * xp[:, u:u + H, v:v + W, :]).sum(axis=(0, 1, 2))
            dxp[:, u:u + H, v:v + W, :] += wdw[:, u, v] * dy
    dx = dxp[:, 1:H + 1, 1:W + 1, :]
    return {"d_o": d_o, "dx": dx, "dw_dw": dw_dw, "db_dw": db_dw, "dw_pw": dw_pw,
            "db_pw": db_pw}
