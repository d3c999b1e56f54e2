"""Pins of the fp64 oracle to things other than itself.

Each test checks an oracle function against a closed form, a brute-force loop
on a tiny window, a library routine in fp64 (torch SDPA / autograd, scipy) or
central finite differences, so that a dropped term, a wrong sign or index or
a transposed operand in the oracle fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def rnd(*shape, std=1.0):
    return rng.standard_normal(shape) * std


# ---------------------------------------------------------------- coordinates

def test_coords_closed_form_m3():
    y, x = O.window_coords(3)
    assert y.tolist() == [-1, -1, -1, 0, 0, 0, 1, 1, 1]
    assert x.tolist() == [-1, 0, 1, -1, 0, 1, -1, 0, 1]


@pytest.mark.parametrize("M", [2, 5, 16, 96])
def test_coords_corners_and_spacing(M):
    y, x = O.window_coords(M)
    # corners of the window sit at (+-1, +-1); steps are 2/(M-1)
    assert (y[0], x[0]) == (-1.0, -1.0)
    assert (y[M - 1], x[M - 1]) == (-1.0, 1.0)
    assert (y[-1], x[-1]) == (1.0, 1.0)
    assert np.allclose(np.diff(x[:M]), 2.0 / (M - 1), atol=1e-15)
    if M % 2 == 1:
        c = (M // 2) * M + M // 2
        assert y[c] == 0.0 and x[c] == 0.0


def test_coords_degenerate_m1():
    y, x = O.window_coords(1)
    assert y.tolist() == [0.0] and x.tolist() == [0.0]


# ---------------------------------------------------------------- Fourier map

def test_fourier_block_order():
    # one frequency w = pi/2, token (y=-1, x=+1)
    g = O.fourier_features(np.array([-1.0]), np.array([1.0]), [math.pi / 2])
    assert np.allclose(g, [[1.0, 0.0, -1.0, 0.0]], atol=1e-15)


def test_fourier_integer_multiples_of_pi_at_edges():
    F = 16
    w = [math.pi * (k + 1) for k in range(F)]
    g = O.fourier_features(np.array([1.0, -1.0]), np.array([-1.0, 1.0]), w)
    signs = np.array([(-1.0) ** (k + 1) for k in range(F)])
    for row in g:
        assert np.allclose(row[0:F], 0.0, atol=1e-13)        # sin(w x)
        assert np.allclose(row[F:2 * F], signs, atol=1e-13)  # cos(w x)
        assert np.allclose(row[2 * F:3 * F], 0.0, atol=1e-13)
        assert np.allclose(row[3 * F:], signs, atol=1e-13)


def test_fourier_unit_circle_and_centre():
    y, x = O.window_coords(7)
    w = rnd(5) * 10
    g = O.fourier_features(y, x, w)
    F = 5
    assert np.allclose(g[:, :F] ** 2 + g[:, F:2 * F] ** 2, 1.0, atol=1e-14)
    assert np.allclose(g[:, 2 * F:3 * F] ** 2 + g[:, 3 * F:] ** 2, 1.0, atol=1e-14)
    c = 3 * 7 + 3                     # centre token of an odd window
    assert np.allclose(g[c], np.r_[np.zeros(F), np.ones(F), np.zeros(F), np.ones(F)])


# ---------------------------------------------------------------- GELU / MLP

def test_gelu_textbook_values():
    # GELU(z) = z * Phi(z); Phi(1), Phi(2) are standard normal table values
    phi1, phi2 = 0.8413447460685429, 0.9772498680518208
    assert abs(O.gelu(1.0) - phi1) < 1e-15
    assert abs(O.gelu(2.0) - 2 * phi2) < 1e-15
    assert abs(O.gelu(-1.0) + (1 - phi1)) < 1e-15
    assert O.gelu(0.0) == 0.0


def test_gelu_matches_torch_exact_gelu():
    z = np.linspace(-6, 6, 101)
    ref = torch.nn.functional.gelu(torch.tensor(z, dtype=torch.float64),
                                   approximate="none").numpy()
    assert np.allclose(O.gelu(z), ref, atol=1e-15, rtol=0)


def test_gelu_grad_finite_difference():
    z = np.linspace(-5, 5, 41)
    h = 1e-6
    fd = (O.gelu(z + h) - O.gelu(z - h)) / (2 * h)
    assert np.allclose(O.gelu_grad(z), fd, atol=1e-8)


def test_mlp_zero_second_layer_gives_bias():
    gam = rnd(10, 8)
    w1, b1 = rnd(6, 8), rnd(6)
    w2, b2 = np.zeros((4, 6)), rnd(4)
    _, _, o = O.mlp_forward(gam, w1, b1, w2, b2)
    assert np.array_equal(o, np.broadcast_to(b2, (10, 4)))


def test_mlp_matches_torch_linear_stack():
    gam = rnd(12, 8)
    w1, b1, w2, b2 = rnd(6, 8), rnd(6), rnd(5, 6), rnd(5)
    t = lambda a: torch.tensor(a, dtype=torch.float64)
    net = torch.nn.Sequential(torch.nn.Linear(8, 6), torch.nn.GELU(),
                              torch.nn.Linear(6, 5)).double()
    with torch.no_grad():
        net[0].weight.copy_(t(w1)); net[0].bias.copy_(t(b1))
        net[2].weight.copy_(t(w2)); net[2].bias.copy_(t(b2))
        ref = net(t(gam)).numpy()
    assert np.allclose(O.mlp_forward(gam, w1, b1, w2, b2)[2], ref, atol=1e-13)


def test_mlp_backward_finite_differences():
    gam = rnd(7, 4)
    params = [rnd(5, 4), rnd(5), rnd(3, 5), rnd(3)]
    g = rnd(7, 3)
    grads = O.mlp_backward(gam, *params, g)

    def loss(ps):
        return float((O.mlp_forward(gam, *ps)[2] * g).sum())

    h = 1e-6
    for pi, p in enumerate(params):
        fd = np.zeros_like(p)
        for idx in np.ndindex(p.shape):
            pp = [q.copy() for q in params]
            pp[pi][idx] += h
            lp = loss(pp)
            pp[pi][idx] -= 2 * h
            lm = loss(pp)
            fd[idx] = (lp - lm) / (2 * h)
        assert np.allclose(grads[pi], fd, rtol=1e-7, atol=1e-8), pi


# ---------------------------------------------------------------- pos tokens

def _mlp(d_in, hid, d_out, std=0.5):
    return (rnd(hid, d_in, std=std), rnd(hid, std=std), rnd(d_out, hid, std=std),
            rnd(d_out, std=std))


def test_pos_tokens_torch_composition():
    """Coordinates -> Fourier -> Linear-GELU-Linear, rebuilt with torch ops."""
    M, heads, r, F, hid = 5, 3, 4, 6, 7
    w = rnd(F) * 3
    mq, mk = _mlp(4 * F, hid, heads * r), _mlp(4 * F, hid, heads * r)
    qp, kp = O.pos_tokens(w, mq, mk, M, heads, r)
    t = lambda a: torch.tensor(a, dtype=torch.float64)
    lin = torch.linspace(-1, 1, M, dtype=torch.float64)
    yy, xx = torch.meshgrid(lin, lin, indexing="ij")
    ang_x = xx.reshape(-1, 1) * t(w)
    ang_y = yy.reshape(-1, 1) * t(w)
    gam = torch.cat([ang_x.sin(), ang_x.cos(), ang_y.sin(), ang_y.cos()], 1)
    for m, got in ((mq, qp), (mk, kp)):
        hdn = torch.nn.functional.gelu(torch.nn.functional.linear(gam, t(m[0]), t(m[1])))
        o = torch.nn.functional.linear(hdn, t(m[2]), t(m[3]))      # [M*M, heads*r]
        ref = o.reshape(M, M, heads, r).permute(2, 0, 1, 3).numpy()
        assert np.allclose(got, ref, atol=1e-13)


def test_pos_tokens_geometry_only_and_param_count_independent_of_window():
    # the same MLP serves every window size; token (i, j) of the window only
    F, heads, r, hid = 4, 2, 3, 5
    w = rnd(F)
    mq, mk = _mlp(4 * F, hid, heads * r), _mlp(4 * F, hid, heads * r)
    for M in (2, 3, 8):
        qp, kp = O.pos_tokens(w, mq, mk, M, heads, r)
        assert qp.shape == (heads, M, M, r) and kp.shape == (heads, M, M, r)
    qp2, _ = O.pos_tokens(w, mq, mk, 2, heads, r)
    qp3, _ = O.pos_tokens(w, mq, mk, 3, heads, r)
    # corners of both windows have the same coordinates -> same tokens
    assert np.allclose(qp2[:, 0, 0], qp3[:, 0, 0]) and np.allclose(qp2[:, 1, 1], qp3[:, 2, 2])


def test_pos_tokens_backward_finite_differences():
    M, heads, r, F, hid = 3, 2, 2, 2, 3
    w = rnd(F)
    mq, mk = list(_mlp(4 * F, hid, heads * r)), list(_mlp(4 * F, hid, heads * r))
    gq, gk = rnd(heads, M, M, r), rnd(heads, M, M, r)
    (dq, dk) = O.pos_tokens_backward(w, mq, mk, M, gq, gk)

    def loss(a, b):
        qp, kp = O.pos_tokens(w, a, b, M, heads, r)
        return float((qp * gq).sum() + (kp * gk).sum())

    h = 1e-6
    for side, grads in ((0, dq), (1, dk)):
        for pi in range(4):
            base = [mq, mk][side]
            fd = np.zeros_like(base[pi])
            for idx in np.ndindex(base[pi].shape):
                for sgn in (+1, -1):
                    pp = [q.copy() for q in base]
                    pp[pi][idx] += sgn * h
                    val = loss(pp, mk) if side == 0 else loss(mq, pp)
                    fd[idx] += sgn * val / (2 * h)
            assert np.allclose(grads[pi], fd, rtol=1e-7, atol=1e-8), (side, pi)


# ---------------------------------------------------------------- scores

@pytest.mark.parametrize("r", [1, 3, 16])
def test_concatenated_dot_product_equals_content_plus_bias(r):
    """The pages' identity [Qc,Qp][Kc,Kp]^T = QcKc^T + QpKp^T, brute force."""
    N, d = 4, 5
    qc, kc, qp, kp = rnd(N, d), rnd(N, d), rnd(N, r), rnd(N, r)
    tau = 0.37
    s = O.unit_scores(qc, kc, qp, kp, tau)
    for t in range(N):
        qa = list(qc[t]) + list(qp[t])
        for u in range(N):
            ka = list(kc[u]) + list(kp[u])
            dot = 0.0
            for a, b in zip(qa, ka):
                dot += a * b
            assert abs(s[t, u] - tau * dot) < 1e-13


# ---------------------------------------------------------------- softmax

def test_attention_two_tokens_is_logistic():
    qc, kc = rnd(2, 3), rnd(2, 3)
    qp, kp = rnd(2, 2), rnd(2, 2)
    v = rnd(2, 4)
    tau = 0.5
    out, lse = O.attention_unit(qc, kc, v, qp, kp, tau)
    for t in range(2):
        s = [tau * (qc[t] @ kc[u] + qp[t] @ kp[u]) for u in range(2)]
        p0 = 1.0 / (1.0 + math.exp(s[1] - s[0]))
        assert np.allclose(out[t], p0 * v[0] + (1 - p0) * v[1], atol=1e-14)
        assert abs(lse[t] - (s[0] + math.log1p(math.exp(s[1] - s[0])))) < 1e-13


def test_attention_rows_sum_to_one_and_lse():
    N, d, r = 37, 6, 3
    qc, kc, qp, kp = rnd(N, d), rnd(N, d), rnd(N, r), rnd(N, r)
    ones = np.ones((N, 1))
    out, lse = O.attention_unit(qc, kc, ones, qp, kp, 0.4)
    assert np.allclose(out, 1.0, atol=1e-14)
    s = 0.4 * (qc @ kc.T + qp @ kp.T)
    assert np.allclose(lse, logsumexp(s, axis=1), atol=1e-13)


def test_zero_queries_give_window_mean():
    N, d, r = 16, 4, 2
    v = rnd(N, d)
    out, lse = O.attention_unit(np.zeros((N, d)), rnd(N, d), v, np.zeros((N, r)),
                                rnd(N, r), 0.3)
    assert np.allclose(out, v.mean(axis=0), atol=1e-14)
    assert np.allclose(lse, math.log(N), atol=1e-14)


@pytest.mark.parametrize("r", [0, 16])
def test_attention_matches_torch_sdpa_augmented(r):
    """Library pin: SDPA on the augmented [Qc,Qp], [Kc,Kp] with its default
    scale 1/sqrt(d+r) equals the oracle with the explicit bias (and, for
    r = 0, plain windowed attention)."""
    N, d = 64, 32
    qc, kc, v = rnd(N, d), rnd(N, d), rnd(N, d)
    qp, kp = rnd(N, r, std=2.0), rnd(N, r, std=2.0)
    out, _ = O.attention_unit(qc, kc, v, qp, kp, O.default_scale(d, r))
    t = lambda a: torch.tensor(a, dtype=torch.float64)[None, None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        t(np.concatenate([qc, qp], 1)), t(np.concatenate([kc, kp], 1)), t(v))[0, 0]
    assert np.allclose(out, ref.numpy(), atol=1e-13)


def test_attention_bias_as_sdpa_float_mask():
    """Library pin of the explicit-bias form S = tau*QcKc^T + tau*B."""
    N, d, r = 50, 8, 4
    qc, kc, v, qp, kp = rnd(N, d), rnd(N, d), rnd(N, d), rnd(N, r), rnd(N, r)
    tau = 0.21
    out, _ = O.attention_unit(qc, kc, v, qp, kp, tau)
    t = lambda a: torch.tensor(a, dtype=torch.float64)
    ref = torch.nn.functional.scaled_dot_product_attention(
        t(qc)[None], t(kc)[None], t(v)[None], attn_mask=t(tau * (qp @ kp.T))[None],
        scale=tau)[0]
    assert np.allclose(out, ref.numpy(), atol=1e-13)


def test_attention_permutation_equivariance():
    N, d, r = 25, 4, 3
    qc, kc, v, qp, kp = rnd(N, d), rnd(N, d), rnd(N, d), rnd(N, r), rnd(N, r)
    perm = rng.permutation(N)
    o1, l1 = O.attention_unit(qc, kc, v, qp, kp, 0.5)
    o2, l2 = O.attention_unit(qc[perm], kc[perm], v[perm], qp[perm], kp[perm], 0.5)
    assert np.allclose(o1[perm], o2, atol=1e-13) and np.allclose(l1[perm], l2, atol=1e-13)


def test_row_blocking_changes_nothing(monkeypatch):
    N, d, r = 300, 4, 2
    args = (rnd(N, d), rnd(N, d), rnd(N, d), rnd(N, r), rnd(N, r), 0.3)
    full = O.attention_unit(*args)
    monkeypatch.setattr(O.rib_oracle, "_ROW_BLOCK", 64)
    blk = O.attention_unit(*args)
    assert np.allclose(full[0], blk[0], atol=1e-14)
    g = rnd(N, d)
    gb = O.attention_unit_backward(*args, g)
    monkeypatch.setattr(O.rib_oracle, "_ROW_BLOCK", 4096)
    gf = O.attention_unit_backward(*args, g)
    for a, b in zip(gb, gf):
        assert np.allclose(a, b, atol=1e-12)


# ---------------------------------------------------------------- partition

def _brute_partition(x, M, s):
    B, H, W = x.shape[:3]
    nW = (H // M) * (W // M)
    out = np.empty((B, nW, M * M) + x.shape[3:], dtype=x.dtype)
    for b, wy, wx, i, j in itertools.product(range(B), range(H // M), range(W // M),
                                             range(M), range(M)):
        out[b, wy * (W // M) + wx, i * M + j] = x[b, (wy * M + i + s) % H,
                                                  (wx * M + j + s) % W]
    return out


@pytest.mark.parametrize("M,s", [(2, 0), (2, 1), (4, 2), (4, 3), (8, 4)])
def test_partition_matches_modular_index_and_inverts(M, s):
    x = rnd(2, 8, 16, 3)
    xw = O.window_partition(x, M, s)
    assert np.array_equal(xw, _brute_partition(x, M, s))
    assert np.array_equal(O.window_reverse(xw, M, s, 8, 16), x)


def test_shift_by_window_multiple_is_same_partition_up_to_window_order():
    x = rnd(1, 8, 8, 2)
    a = O.window_partition(x, 4, 1)
    b = O.window_partition(x, 4, 5)
    # s+M shifts by one whole window: the same windows, relabelled
    assert sorted(map(lambda w: w.tobytes(), a[0])) == sorted(map(lambda w: w.tobytes(), b[0]))


def test_full_map_shift_invariance_under_window_multiple():
    B, H, W, heads, d, M, r = 1, 8, 8, 2, 3, 4, 2
    qkv = rnd(B, H, W, 3, heads, d)
    qp, kp = rnd(heads, M, M, r), rnd(heads, M, M, r)
    o1, l1 = O.attn_fwd(qkv, M, 1, qp, kp)
    o2, l2 = O.attn_fwd(qkv, M, 1 + M, qp, kp)
    assert np.allclose(o1, o2, atol=1e-14) and np.allclose(l1, l2, atol=1e-14)


def test_full_map_against_per_pixel_brute_force():
    B, H, W, heads, d, M, r, s = 1, 4, 6, 2, 3, 2, 2, 1
    qkv = rnd(B, H, W, 3, heads, d)
    qp, kp = rnd(heads, M, M, r), rnd(heads, M, M, r)
    tau = 0.6
    out, lse = O.attn_fwd(qkv, M, s, qp, kp, tau)
    # every pixel attends to the pixels of its rolled window; tokens are
    # identified by their window-local (i, j)
    for y, x, h in itertools.product(range(H), range(W), range(heads)):
        yr, xr = (y - s) % H, (x - s) % W          # position after roll(-s)
        wy, wx, i, j = yr // M, xr // M, yr % M, xr % M
        logits, vals = [], []
        for a, b in itertools.product(range(M), range(M)):
            py, px = (wy * M + a + s) % H, (wx * M + b + s) % W
            dot = qkv[0, y, x, 0, h] @ qkv[0, py, px, 1, h] + qp[h, i, j] @ kp[h, a, b]
            logits.append(tau * dot)
            vals.append(qkv[0, py, px, 2, h])
        p = np.exp(np.array(logits) - max(logits))
        ref = (p[:, None] * np.array(vals)).sum(0) / p.sum()
        assert np.allclose(out[0, y, x, h], ref, atol=1e-13)
        assert abs(lse[0, h, y, x] - logsumexp(logits)) < 1e-13


# ---------------------------------------------------------------- backward

def _tiny_problem():
    B, H, W, heads, d, M, r, s = 1, 4, 4, 2, 3, 2, 2, 1
    return (rnd(B, H, W, 3, heads, d), rnd(heads, M, M, r), rnd(heads, M, M, r),
            rnd(B, H, W, heads, d), M, s)


def test_attn_bwd_finite_differences():
    qkv, qp, kp, g, M, s = _tiny_problem()
    tau = 0.45
    dqkv, dqp, dkp = O.attn_bwd(qkv, g, M, s, qp, kp, tau)

    def loss(a, b, c):
        return float((O.attn_fwd(a, M, s, b, c, tau)[0] * g).sum())

    h = 1e-6
    for arr, grad, pos in ((qkv, dqkv, 0), (qp, dqp, 1), (kp, dkp, 2)):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            vals = []
            for sgn in (+1, -1):
                args = [qkv.copy(), qp.copy(), kp.copy()]
                args[pos][idx] += sgn * h
                vals.append(loss(*args))
            fd[idx] = (vals[0] - vals[1]) / (2 * h)
        assert np.allclose(grad, fd, rtol=1e-6, atol=1e-8), pos


def test_attn_bwd_matches_torch_autograd():
    B, H, W, heads, d, M, r, s = 2, 8, 8, 2, 5, 4, 3, 2
    qkv = rnd(B, H, W, 3, heads, d)
    qp, kp = rnd(heads, M, M, r), rnd(heads, M, M, r)
    g = rnd(B, H, W, heads, d)
    tau = O.default_scale(d, r)
    dqkv, dqp, dkp = O.attn_bwd(qkv, g, M, s, qp, kp)
    tq = torch.tensor(qkv, requires_grad=True)
    tqp = torch.tensor(qp, requires_grad=True)
    tkp = torch.tensor(kp, requires_grad=True)
    x = torch.roll(tq, (-s, -s), (1, 2)).reshape(B, H // M, M, W // M, M, 3, heads, d)
    x = x.permute(0, 1, 3, 6, 2, 4, 5, 7).reshape(B, -1, heads, M * M, 3, d)
    q = torch.cat([x[..., 0, :], tqp.reshape(heads, M * M, r).expand(B, x.shape[1], -1, -1, -1)], -1)
    k = torch.cat([x[..., 1, :], tkp.reshape(heads, M * M, r).expand(B, x.shape[1], -1, -1, -1)], -1)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, x[..., 2, :])
    o = o.reshape(B, H // M, W // M, heads, M, M, d).permute(0, 1, 4, 2, 5, 3, 6)
    o = torch.roll(o.reshape(B, H, W, heads, d), (s, s), (1, 2))
    (o * torch.tensor(g)).sum().backward()
    assert np.allclose(dqkv, tq.grad.numpy(), atol=1e-12)
    assert np.allclose(dqp, tqp.grad.numpy(), atol=1e-12)
    assert np.allclose(dkp, tkp.grad.numpy(), atol=1e-12)
    assert abs(tau - 1 / math.sqrt(d + r)) < 1e-16


def test_key_gradients_sum_to_zero():
    """Rows of dS = P*(dP - rowsum(P*dP)) sum to zero, so sum_k dK[k] = 0 for
    both the content and the positional key gradients."""
    N, d, r = 40, 6, 3
    g = O.attention_unit_backward(rnd(N, d), rnd(N, d), rnd(N, d), rnd(N, r), rnd(N, r), 0.7,
                                  rnd(N, d))
    dkc, dkp = g[1], g[4]
    assert np.allclose(dkc.sum(0), 0, atol=1e-12 * np.abs(dkc).sum())
    assert np.allclose(dkp.sum(0), 0, atol=1e-12 * np.abs(dkp).sum())


def test_attn_bwd_unit_subset_equals_zero_upstream_elsewhere():
    qkv, qp, kp, g, M, s = _tiny_problem()
    keep = {(0, 1, 0), (0, 3, 1)}
    sub = O.attn_bwd(qkv, g, M, s, qp, kp, units=keep)
    # zero the upstream gradient of every other unit's tokens
    gw = O.window_partition(g, M, s)
    for b, w, h in itertools.product(range(1), range(4), range(2)):
        if (b, w, h) not in keep:
            gw[b, w, :, h] = 0
    g0 = O.window_reverse(gw, M, s, 4, 4)
    full = O.attn_bwd(qkv, g0, M, s, qp, kp)
    for a, b in zip(sub, full):
        assert np.allclose(a, b, atol=1e-14)


# ---------------------------------------------------------------- golden

def test_golden_closed_forms():
    with open(os.path.join(GOLDEN, "closed_forms.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        a = {k: np.array(v, dtype=np.float64) for k, v in c["inputs"].items()}
        out, lse = O.attention_unit(a["qc"], a["kc"], a["v"], a["qp"], a["kp"],
                                    c["scale"])
        assert np.allclose(out, c["expect"]["out"], atol=1e-12), c["name"]
        assert np.allclose(lse, c["expect"]["lse"], atol=1e-12), c["name"]


# ---------------------------------------------------------------- unit helpers

def _brute_unit(qkv, qp, kp, M, s, b, w, h):
    """Unit (b, w, h) read pixel by pixel: token t = i*M + j of window
    w = wy*(W/M) + wx sits at map pixel ((wy*M+i+s) mod H, (wx*M+j+s) mod W)
    (the roll by -s, then the partition); its position tokens are row (i, j)
    of head h."""
    H, W = qkv.shape[1:3]
    wy, wx = divmod(w, W // M)
    N = M * M
    d, r = qkv.shape[-1], qp.shape[-1]
    qc, kc, v = np.empty((N, d)), np.empty((N, d)), np.empty((N, d))
    qpu, kpu = np.empty((N, r)), np.empty((N, r))
    for i, j in itertools.product(range(M), range(M)):
        t = i * M + j
        y, x = (wy * M + i + s) % H, (wx * M + j + s) % W
        qc[t], kc[t], v[t] = qkv[b, y, x, 0, h], qkv[b, y, x, 1, h], qkv[b, y, x, 2, h]
        qpu[t], kpu[t] = qp[h, i, j], kp[h, i, j]
    return qc, kc, v, qpu, kpu


@pytest.mark.parametrize("M,s,b,w,h", [(2, 1, 1, 5, 2), (4, 2, 0, 3, 1), (4, 0, 1, 0, 0),
                                       (4, 3, 1, 2, 2)])
def test_gather_unit_matches_pixel_index(M, s, b, w, h):
    B, H, W, heads, d, r = 2, 8, 12, 3, 5, 2
    qkv = rnd(B, H, W, 3, heads, d)
    qp, kp = rnd(heads, M, M, r), rnd(heads, M, M, r)
    got = O.gather_unit(qkv, qp, kp, M, s, b, w, h)
    want = _brute_unit(qkv, qp, kp, M, s, b, w, h)
    for g, e in zip(got, want):
        assert np.array_equal(g, e)


def test_gather_unit_then_attention_is_the_map_output():
    """The unit read by gather_unit, attended, lands at the map pixels that
    attn_fwd (checked pixel by pixel above) writes for that unit."""
    B, H, W, heads, d, M, r, s = 2, 8, 8, 2, 3, 4, 2, 2
    qkv = rnd(B, H, W, 3, heads, d)
    qp, kp = rnd(heads, M, M, r), rnd(heads, M, M, r)
    tau = 0.4
    out, lse = O.attn_fwd(qkv, M, s, qp, kp, tau)
    for b, w, h in ((1, 3, 1), (0, 1, 0)):
        o, l = O.attention_unit(*O.gather_unit(qkv, qp, kp, M, s, b, w, h), tau)
        wy, wx = divmod(w, W // M)
        for i, j in itertools.product(range(M), range(M)):
            y, x = (wy * M + i + s) % H, (wx * M + j + s) % W
            assert np.allclose(out[b, y, x, h], o[i * M + j], atol=1e-14)
            assert abs(lse[b, h, y, x] - l[i * M + j]) < 1e-14


def _brute_rows(qc, kc, v, qp, kp, tau, rows, labels):
    """Each requested query row on its own: scores over the keys it may see
    (all, or those sharing its region label), softmax, weighted sum of V."""
    outs, lses = [], []
    for t in rows:
        keys = [u for u in range(kc.shape[0]) if labels is None or labels[u] == labels[t]]
        logits = np.array([tau * (qc[t] @ kc[u] + qp[t] @ kp[u]) for u in keys])
        p = np.exp(logits - logits.max())
        outs.append((p[:, None] * v[keys]).sum(0) / p.sum())
        lses.append(logsumexp(logits))
    return np.array(outs), np.array(lses)


@pytest.mark.parametrize("masked", [False, True])
def test_attention_unit_rows_matches_per_row_brute_force(monkeypatch, masked):
    """A row subset that is unsorted, repeats a row and, with a small row
    block, straddles block edges and every region band of a corner window."""
    H = W = 32
    M, s = 16, 8
    N, d, r = M * M, 4, 3
    qc, kc, v, qp, kp = rnd(N, d), rnd(N, d), rnd(N, d), rnd(N, r), rnd(N, r)
    lab = O.region_labels(H, W, M, s, 1, 1) if masked else None
    if masked:
        assert len(set(lab.tolist())) == 4
    rows = np.array([255, 0, 7, 8, 9, 120, 136, 17, 250, 8, 64, 191])
    monkeypatch.setattr(O.rib_oracle, "_ROW_BLOCK", 5)
    out, lse = O.attention_unit_rows(qc, kc, v, qp, kp, 0.35, rows=rows, labels=lab)
    ref_o, ref_l = _brute_rows(qc, kc, v, qp, kp, 0.35, rows, lab)
    assert out.shape == (len(rows), d)
    assert np.allclose(out, ref_o, atol=1e-13)
    assert np.allclose(lse, ref_l, atol=1e-13)
