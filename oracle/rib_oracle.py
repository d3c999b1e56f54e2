"""Plain fp64 CPU oracle for RIB windowed attention (TEST INFRASTRUCTURE ONLY).

Only the test-suite, the package's smoke check and the CPU-baseline leg of the
benchmark may import this module.  The product path never calls it; it shares
no code, table or helper with the CUDA library.

Sources (web pages about arXiv 2603.06738, "Rank-Factorized Implicit Neural
Bias: Scaling Super-Resolution Transformer with FlashAttention"), cited below
by short tag:

  [ABS] the paper's abstract (khansong-paper-with-me.hf.space)
  [EN]  gist.science English summary, Technical Summary
  [DE]  gist.science/de German summary, Methodik
  [ZH]  gist.science/zh Chinese summary, 核心方法论
  [ES]  gist.science/es Spanish summary, Metodología

What the pages fix:
  * every token gets a normalised 2D coordinate in [-1, 1] that goes through
    a Fourier feature map ([DE] §A step 1, [EN] §2.A step 1, [ZH] §2.A 1);
  * a lightweight MLP maps it to low-rank positional tokens Qp, Kp
    ([EN] §2.A step 2, [DE] §A step 2);
  * Qp, Kp are concatenated channel-wise with the content tokens Qc, Kc and
    the score is the single dot product [Qc,Qp][Kc,Kp]^T = QcKc^T + QpKp^T
    ([EN] §2.A steps 3-4 and its score equation, [ABS]);
  * the bias replaces the explicit form S = QK^T + B ([EN] §2.A Mechanism),
    which this oracle computes literally: it materialises B = Qp Kp^T;
  * Qp/Kp depend only on window geometry and can be cached ([ZH] §2.A, [DE]).

Readings where the pages are silent (each is an argument of a function here,
so a test can vary it):
  1. coordinates are local to the window, endpoints included:
     y_i = -1 + 2i/(M-1), x_j = -1 + 2j/(M-1);
  2. Fourier features [sin(w x), cos(w x), sin(w y), cos(w y)] over the given
     angular frequencies w (default pi*(k+1), k<16), 4F = 64 inputs;
  3. two MLPs (one for Qp, one for Kp): Linear -> GELU(erf form) -> Linear,
     output column o = head*rank + r;
  4. softmax scale tau applied to the whole augmented product, default
     1/sqrt(d + rank);
  5. the window shift is a pure cyclic roll by -s on both map axes before the
     partition and +s after it, with no region mask.  An optional variant
     (off by default, `region_mask=True`) adds the usual shifted-window
     region mask, which the pages do not describe: on the rolled map, rows
     split into [0, H-M), [H-M, H-s), [H-s, H) and columns likewise, and a
     query attends only to keys of its own (row band, column band) region;
  6. lse is the natural-log log-sum-exp of the scaled scores.

Memory: rows of the N x N score matrix are processed in row blocks when N is
large; every row's softmax is independent, so a block changes no row's
arithmetic, and the key-side gradient sums still run over every row.

Pins: every function here is checked, in tests/test_oracle_pins.py and
tests/test_region_mask_oracle.py, against closed forms, brute force on tiny
windows (the unit read pixel by pixel through the modular roll index, each
requested query row attended on its own), library routines (torch SDPA and
autograd in fp64) and central finite differences; tests/test_oracle_mutations.py
plants a plausible mistake in each and checks that a pin fails.  No function
is "parity unpinned".
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf

__all__ = [
    "window_coords", "fourier_features", "gelu", "gelu_grad", "mlp_forward",
    "mlp_backward", "pos_tokens", "pos_tokens_backward", "window_partition",
    "window_reverse", "unit_scores", "attention_unit", "attention_unit_rows",
    "attention_unit_backward", "attn_fwd", "attn_bwd", "default_scale",
    "gather_unit", "region_labels",
]

_ROW_BLOCK = 2048


def _f64(a):
    """Host array as fp64 numpy (accepts torch tensors of any dtype)."""
    if hasattr(a, "detach"):
        a = a.detach().cpu()
        if str(a.dtype) in ("torch.bfloat16", "torch.float16"):
            a = a.float()
        a = a.numpy()
    return np.asarray(a, dtype=np.float64)


def default_scale(head_dim: int, rank: int) -> float:
    """Reading 4: tau = 1/sqrt(d + r), the scale of the augmented product."""
    return 1.0 / np.sqrt(head_dim + rank)


# --------------------------------------------------------------------------
# Position tokens: coordinates -> Fourier features -> MLP -> Qp, Kp
# --------------------------------------------------------------------------

def window_coords(M: int):
    """Normalised window coordinates of the M*M tokens, row-major t = i*M+j.

    [DE] §A step 1: each token gets a normalised 2D coordinate in [-1, 1].
    Reading 1: local to the window, endpoints included.  Returns (y, x), each
    [M*M] fp64; M == 1 gives the single coordinate (0, 0)."""
    if M == 1:
        lin = np.zeros(1)
    else:
        lin = -1.0 + 2.0 * np.arange(M, dtype=np.float64) / (M - 1)
    y = np.repeat(lin, M)      # row index i varies slowest
    x = np.tile(lin, M)        # column index j varies fastest
    return y, x


def fourier_features(y, x, freqs):
    """Fourier feature map of the coordinates ([EN] §2.A step 1).

    Reading 2: gamma = [sin(w x), cos(w x), sin(w y), cos(w y)], each block
    over the F given angular frequencies w.  Returns [N, 4F] fp64."""
    w = _f64(freqs).reshape(1, -1)
    ax = np.asarray(x, dtype=np.float64).reshape(-1, 1) * w
    ay = np.asarray(y, dtype=np.float64).reshape(-1, 1) * w
    return np.concatenate([np.sin(ax), np.cos(ax), np.sin(ay), np.cos(ay)],
                          axis=1)


def gelu(z):
    """GELU, erf form: z * Phi(z)."""
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + erf(z / np.sqrt(2.0)))


def gelu_grad(z):
    """d/dz GELU(z) = Phi(z) + z * phi(z)."""
    z = np.asarray(z, dtype=np.float64)
    cdf = 0.5 * (1.0 + erf(z / np.sqrt(2.0)))
    pdf = np.exp(-0.5 * z * z) / np.sqrt(2.0 * np.pi)
    return cdf + z * pdf


def mlp_forward(gamma, w1, b1, w2, b2):
    """Lightweight MLP of [EN] §2.A step 2 (reading 3: Linear-GELU-Linear).

    gamma [N, d_in]; w1 [hid, d_in]; w2 [d_out, hid] (PyTorch Linear layout).
    Returns (pre-activation a, hidden h, output o)."""
    a = gamma @ _f64(w1).T + _f64(b1)
    h = gelu(a)
    o = h @ _f64(w2).T + _f64(b2)
    return a, h, o


def mlp_backward(gamma, w1, b1, w2, b2, d_out):
    """Gradients of sum(mlp_forward(...)[2] * d_out) w.r.t. w1, b1, w2, b2.

    Chain rule through the two Linear layers and GELU."""
    a, h, _ = mlp_forward(gamma, w1, b1, w2, b2)
    g = _f64(d_out)
    dw2 = g.T @ h
    db2 = g.sum(axis=0)
    dh = g @ _f64(w2)
    da = dh * gelu_grad(a)
    dw1 = da.T @ gamma
    db1 = da.sum(axis=0)
    return dw1, db1, dw2, db2


def _mlp_tuple(m):
    if isinstance(m, (tuple, list)):
        return m
    return (m.w1, m.b1, m.w2, m.b2)


def pos_tokens(freqs, mlp_q, mlp_k, M: int, heads: int, rank: int):
    """Positional tokens Qp, Kp for an M x M window, fp64 [heads][M][M][rank].

    Coordinates -> Fourier features -> one MLP per side ([EN] §2.A steps 1-2).
    They depend only on the window geometry ([ZH] §2.A), so one set serves
    every window, batch entry and layer with the same M and weights."""
    y, x = window_coords(M)
    gam = fourier_features(y, x, freqs)
    out = []
    for m in (mlp_q, mlp_k):
        _, _, o = mlp_forward(gam, *_mlp_tuple(m))
        assert o.shape[1] == heads * rank
        out.append(o.reshape(M, M, heads, rank).transpose(2, 0, 1, 3).copy())
    return out[0], out[1]


def pos_tokens_backward(freqs, mlp_q, mlp_k, M: int, dqp, dkp):
    """MLP weight gradients given dL/dQp and dL/dKp ([heads][M][M][rank]).

    Returns ((dw1,db1,dw2,db2) for the q MLP, (...) for the k MLP)."""
    y, x = window_coords(M)
    gam = fourier_features(y, x, freqs)
    res = []
    for m, d in ((mlp_q, dqp), (mlp_k, dkp)):
        d = _f64(d)
        heads, _, _, rank = d.shape
        g = d.transpose(1, 2, 0, 3).reshape(M * M, heads * rank)
        res.append(mlp_backward(gam, *_mlp_tuple(m), g))
    return tuple(res)


# --------------------------------------------------------------------------
# Window partition with cyclic shift
# --------------------------------------------------------------------------

def window_partition(x, M: int, s: int):
    """x [B, H, W, ...] -> [B, nW, M*M, ...] after a cyclic roll by -s.

    Reading 5: roll both map axes by -s, then cut M x M windows; window index
    wy*(W/M)+wx, token index i*M+j inside the window."""
    x = np.asarray(x)
    B, H, W = x.shape[:3]
    rest = x.shape[3:]
    xr = np.roll(x, shift=(-s, -s), axis=(1, 2))
    xr = xr.reshape((B, H // M, M, W // M, M) + rest)
    xr = np.moveaxis(xr, 3, 2)           # B, H/M, W/M, M, M, ...
    return xr.reshape((B, (H // M) * (W // M), M * M) + rest)


def window_reverse(xw, M: int, s: int, H: int, W: int):
    """Exact inverse of window_partition: un-partition, then roll by +s."""
    xw = np.asarray(xw)
    B = xw.shape[0]
    rest = xw.shape[3:]
    x = xw.reshape((B, H // M, W // M, M, M) + rest)
    x = np.moveaxis(x, 2, 3)             # B, H/M, M, W/M, M, ...
    x = x.reshape((B, H, W) + rest)
    return np.roll(x, shift=(s, s), axis=(1, 2))


# --------------------------------------------------------------------------
# Attention for one (batch, window, head) unit
# --------------------------------------------------------------------------

def region_labels(H: int, W: int, M: int, s: int, wy: int, wx: int):
    """Region label of each token of window (wy, wx), [M*M] ints, t = i*M+j.

    Reading 5's optional mask: on the map rolled by -s, a row y belongs to
    band 0 if y < H-M, band 1 if y < H-s, else band 2 (columns alike with W);
    the label is 3*row_band + column_band.  With s = 0 every label is 0."""
    def band(pos, size):
        if s == 0:
            return np.zeros_like(pos)
        return np.where(pos < size - M, 0, np.where(pos < size - s, 1, 2))
    i, j = np.divmod(np.arange(M * M), M)
    return 3 * band(wy * M + i, H) + band(wx * M + j, W)


def unit_scores(qc, kc, qp, kp, scale, allowed=None):
    """Scaled scores S = tau * (Qc Kc^T + B) with the explicit bias B = Qp Kp^T.

    This is the RPB-style form S = QK^T + B of [EN] §2.A (Mechanism) with the
    bias materialised; the pages' identity says it equals the augmented dot
    product, which the pins check separately.  `allowed` (bool [rows, keys]),
    if given, sets the scores of the other pairs to -inf."""
    bias = _f64(qp) @ _f64(kp).T
    sc = scale * (_f64(qc) @ _f64(kc).T + bias)
    if allowed is not None:
        sc = np.where(allowed, sc, -np.inf)
    return sc


def _softmax_rows(s):
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    return e / l, (m + np.log(l))[:, 0]


def _allowed(labels, r0, r1, rows=None):
    """Query rows r0..r1 (of `rows`, if given) x all keys: same region label."""
    if labels is None:
        return None
    q = labels[rows][r0:r1] if rows is not None else labels[r0:r1]
    return q[:, None] == labels[None, :]


def attention_unit_rows(qc, kc, v, qp, kp, scale, rows=None, labels=None):
    """Output and lse of the given query rows of one unit (all rows if None).

    softmax over keys of tau*(Qc Kc^T + Qp Kp^T), then P V.  With `labels`
    (region label per token, see region_labels) a query only sees keys of its
    own label."""
    qc, kc, v, qp, kp = map(_f64, (qc, kc, v, qp, kp))
    if rows is not None:
        qc, qp = qc[rows], qp[rows]
    n = qc.shape[0]
    out = np.empty((n, v.shape[1]))
    lse = np.empty(n)
    for r0 in range(0, n, _ROW_BLOCK):
        r1 = min(n, r0 + _ROW_BLOCK)
        s = unit_scores(qc[r0:r1], kc, qp[r0:r1], kp, scale, _allowed(labels, r0, r1, rows))
        p, lse[r0:r1] = _softmax_rows(s)
        out[r0:r1] = p @ v
    return out, lse


def attention_unit(qc, kc, v, qp, kp, scale, labels=None):
    """Forward of one unit: (O [N, d], lse [N])."""
    return attention_unit_rows(qc, kc, v, qp, kp, scale, labels=labels)


def attention_unit_backward(qc, kc, v, qp, kp, scale, dout, labels=None):
    """Textbook softmax-attention backward of one unit, fp64.

    With P = softmax(S), O = P V and upstream dO:
      dV = P^T dO,  dP = dO V^T,  dS = P * (dP - rowsum(P * dP)),
      dQc = tau dS Kc,  dQp = tau dS Kp,  dKc = tau dS^T Qc,  dKp = tau dS^T Qp
    (the bias term tau*Qp Kp^T contributes the Qp/Kp gradients).  Masked
    pairs (`labels`) have P = 0, hence dS = 0."""
    qc, kc, v, qp, kp, do = map(_f64, (qc, kc, v, qp, kp, dout))
    n = qc.shape[0]
    dqc = np.empty_like(qc)
    dqp = np.empty_like(qp)
    dkc = np.zeros_like(kc)
    dkp = np.zeros_like(kp)
    dv = np.zeros_like(v)
    for r0 in range(0, n, _ROW_BLOCK):
        r1 = min(n, r0 + _ROW_BLOCK)
        s = unit_scores(qc[r0:r1], kc, qp[r0:r1], kp, scale, _allowed(labels, r0, r1))
        p, _ = _softmax_rows(s)
        dob = do[r0:r1]
        dv += p.T @ dob
        dp = dob @ v.T
        ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
        dqc[r0:r1] = scale * (ds @ kc)
        dqp[r0:r1] = scale * (ds @ kp)
        dkc += scale * (ds.T @ qc[r0:r1])
        dkp += scale * (ds.T @ qp[r0:r1])
    return dqc, dkc, dv, dqp, dkp


def gather_unit(qkv, qp, kp, M, s, b, w, h):
    """Qc, Kc, V [N, d] of unit (b, window w, head h) and its Qp, Kp [N, r]."""
    x = _f64(qkv)[b:b + 1]
    xw = window_partition(x, M, s)[0, w]          # [N, 3, heads, d]
    qpf = _f64(qp)[h].reshape(M * M, -1)
    kpf = _f64(kp)[h].reshape(M * M, -1)
    return xw[:, 0, h], xw[:, 1, h], xw[:, 2, h], qpf, kpf


# --------------------------------------------------------------------------
# Whole feature map
# --------------------------------------------------------------------------

def attn_fwd(qkv, M: int, s: int, qp, kp, scale=None, region_mask=False):
    """Windowed RIB attention over a feature map.

    qkv [B][H][W][3][heads][d] (Qc, Kc, V); qp, kp [heads][M][M][r].
    Returns out [B][H][W][heads][d] and lse [B][heads][H][W], both fp64, at
    the original (un-rolled) pixel positions.  region_mask: reading 5's
    optional shifted-window mask."""
    x = _f64(qkv)
    B, H, W, _, heads, d = x.shape
    r = _f64(qp).shape[-1]
    if scale is None:
        scale = default_scale(d, r)
    xw = window_partition(x, M, s)                # [B, nW, N, 3, heads, d]
    nW = xw.shape[1]
    ow = np.empty((B, nW, M * M, heads, d))
    lw = np.empty((B, nW, M * M, heads))
    for h in range(heads):
        qpf = _f64(qp)[h].reshape(M * M, r)
        kpf = _f64(kp)[h].reshape(M * M, r)
        for b in range(B):
            for w in range(nW):
                lab = (region_labels(H, W, M, s, w // (W // M), w % (W // M))
                       if region_mask else None)
                o, l = attention_unit(xw[b, w, :, 0, h], xw[b, w, :, 1, h],
                                      xw[b, w, :, 2, h], qpf, kpf, scale, labels=lab)
                ow[b, w, :, h] = o
                lw[b, w, :, h] = l
    out = window_reverse(ow, M, s, H, W)
    lse = window_reverse(lw, M, s, H, W).transpose(0, 3, 1, 2)
    return out, lse


def attn_bwd(qkv, dout, M: int, s: int, qp, kp, scale=None, units=None, region_mask=False):
    """Gradients of sum(attn_fwd(...)[0] * dout).

    Returns dqkv [B][H][W][3][heads][d] and dqp, dkp [heads][M][M][r] summed
    over batch entries and windows.  `units`, if given, is a set of
    (b, w, h) triples; the other units are skipped (their dout is taken as 0),
    which the full-size sampled parity checks use."""
    x = _f64(qkv)
    B, H, W, _, heads, d = x.shape
    r = _f64(qp).shape[-1]
    if scale is None:
        scale = default_scale(d, r)
    xw = window_partition(x, M, s)
    dow = window_partition(_f64(dout), M, s)
    nW = xw.shape[1]
    dxw = np.zeros_like(xw)
    dqp = np.zeros((heads, M * M, r))
    dkp = np.zeros((heads, M * M, r))
    for h in range(heads):
        qpf = _f64(qp)[h].reshape(M * M, r)
        kpf = _f64(kp)[h].reshape(M * M, r)
        for b in range(B):
            for w in range(nW):
                if units is not None and (b, w, h) not in units:
                    continue
                lab = (region_labels(H, W, M, s, w // (W // M), w % (W // M))
                       if region_mask else None)
                g = attention_unit_backward(
                    xw[b, w, :, 0, h], xw[b, w, :, 1, h], xw[b, w, :, 2, h],
                    qpf, kpf, scale, dow[b, w, :, h], labels=lab)
                dxw[b, w, :, 0, h] = g[0]
                dxw[b, w, :, 1, h] = g[1]
                dxw[b, w, :, 2, h] = g[2]
                dqp[h] += g[3]
                dkp[h] += g[4]
    dqkv = window_reverse(dxw, M, s, H, W)
    return (dqkv, dqp.reshape(heads, M, M, r), dkp.reshape(heads, M, M, r))
