"""Pins of the CLA gate oracle (oracle/cla_oracle.py) to things other than
itself: torch's fp64 conv2d, closed forms, special cases and central finite
differences (no GPU)."""
import numpy as np
import pytest
import torch

import oracle as O


def _rand(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape) * scale


def _params(C, seed):
    return (_rand((C, 3, 3), seed, 0.5), _rand((C,), seed + 1, 0.3),
            _rand((C, C), seed + 2, 0.7 / np.sqrt(C)), _rand((C,), seed + 3, 0.3))


def test_dw_conv_matches_torch_grouped_conv2d_fp64():
    B, H, W, C = 2, 5, 7, 4
    x = _rand((B, H, W, C), 0)
    w, b, _, _ = _params(C, 10)
    ref = torch.nn.functional.conv2d(torch.from_numpy(x).permute(0, 3, 1, 2),
                                     torch.from_numpy(w)[:, None], torch.from_numpy(b),
                                     padding=1, groups=C).permute(0, 2, 3, 1).numpy()
    np.testing.assert_allclose(O.dw_conv3x3(x, w, b), ref, rtol=0, atol=1e-13)


def test_pw_conv_matches_torch_1x1_conv2d_fp64():
    B, H, W, C = 1, 3, 4, 6
    y = _rand((B, H, W, C), 1)
    _, _, w, b = _params(C, 20)
    ref = torch.nn.functional.conv2d(torch.from_numpy(y).permute(0, 3, 1, 2),
                                     torch.from_numpy(w)[:, :, None, None],
                                     torch.from_numpy(b)).permute(0, 2, 3, 1).numpy()
    np.testing.assert_allclose(O.pw_conv(y, w, b), ref, rtol=0, atol=1e-13)


def test_sigmoid_closed_forms():
    np.testing.assert_allclose(O.sigmoid(np.array([0.0, np.log(3.0), -np.log(3.0)])),
                               [0.5, 0.75, 0.25], rtol=0, atol=1e-15)


def test_zero_pointwise_weight_gives_constant_gate():
    B, H, W, C = 1, 4, 4, 3
    x = _rand((B, H, W, C), 2)
    w_dw, b_dw, _, b_pw = _params(C, 30)
    g = O.cla_gate(x, w_dw, b_dw, np.zeros((C, C)), b_pw)
    np.testing.assert_allclose(g, np.broadcast_to(1 / (1 + np.exp(-b_pw)), g.shape), atol=1e-15)


def test_interior_impulse_spreads_the_kernel_by_cross_correlation():
    C, H, W = 2, 7, 7
    x = np.zeros((1, H, W, C))
    x[0, 3, 4, 1] = 1.0
    w = _rand((C, 3, 3), 3)
    y = O.dw_conv3x3(x, w, np.zeros(C))
    # y[i, j] = sum_{u,v} w[u, v] x[i+u-1, j+v-1]: the impulse at (3, 4) is
    # seen by output (3-u+1, 4-v+1) through tap (u, v)
    for u in range(3):
        for v in range(3):
            assert y[0, 3 - u + 1, 4 - v + 1, 1] == w[1, u, v]
    assert np.count_nonzero(y[..., 0]) == 0
    assert np.count_nonzero(y[..., 1]) == np.count_nonzero(w[1])


def test_gate_application_with_saturated_gate_is_identity():
    o = _rand((1, 2, 3, 4), 4)
    np.testing.assert_array_equal(O.cla_apply(o, np.ones_like(o)), o)
    np.testing.assert_array_equal(O.cla_apply(o, np.zeros_like(o)), np.zeros_like(o))


def _loss(x, w_dw, b_dw, w_pw, b_pw, o, dout):
    return float((O.cla_apply(o, O.cla_gate(x, w_dw, b_dw, w_pw, b_pw)) * dout).sum())


@pytest.mark.parametrize("name", ["x", "w_dw", "b_dw", "w_pw", "b_pw", "o"])
def test_backward_matches_central_finite_differences(name):
    B, H, W, C = 1, 4, 5, 3
    args = dict(x=_rand((B, H, W, C), 5), o=_rand((B, H, W, C), 6))
    args["w_dw"], args["b_dw"], args["w_pw"], args["b_pw"] = _params(C, 40)
    dout = _rand((B, H, W, C), 7)
    g = O.cla_backward(args["x"], args["w_dw"], args["b_dw"], args["w_pw"], args["b_pw"],
                       args["o"], dout)
    key = {"x": "dx", "w_dw": "dw_dw", "b_dw": "db_dw", "w_pw": "dw_pw", "b_pw": "db_pw",
           "o": "d_o"}[name]
    base = args[name]
    num = np.zeros_like(base)
    h = 1e-6
    for idx in np.ndindex(base.shape):
        save = base[idx]
        base[idx] = save + h
        lp = _loss(dout=dout, **args)
        base[idx] = save - h
        lm = _loss(dout=dout, **args)
        base[idx] = save
        num[idx] = (lp - lm) / (2 * h)
    an = g[key].reshape(num.shape)
    assert np.abs(an - num).max() <= 1e-7 * max(1.0, np.abs(num).max())


def test_backward_matches_torch_autograd_fp64():
    B, H, W, C = 2, 3, 4, 5
    x = _rand((B, H, W, C), 8)
    o = _rand((B, H, W, C), 9)
    dout = _rand((B, H, W, C), 11)
    w_dw, b_dw, w_pw, b_pw = _params(C, 50)
    t = {k: torch.tensor(v, requires_grad=True) for k, v in
         dict(x=x, w_dw=w_dw, b_dw=b_dw, w_pw=w_pw, b_pw=b_pw, o=o).items()}
    y = torch.nn.functional.conv2d(t["x"].permute(0, 3, 1, 2), t["w_dw"][:, None], t["b_dw"],
                                   padding=1, groups=C)
    z = torch.nn.functional.conv2d(y, t["w_pw"][:, :, None, None], t["b_pw"])
    out = t["o"] * torch.sigmoid(z).permute(0, 2, 3, 1)
    (out * torch.from_numpy(dout)).sum().backward()
    g = O.cla_backward(x, w_dw, b_dw, w_pw, b_pw, o, dout)
    for k, name in (("dx", "x"), ("dw_dw", "w_dw"), ("db_dw", "b_dw"), ("dw_pw", "w_pw"),
                    ("db_pw", "b_pw"), ("d_o", "o")):
        np.testing.assert_allclose(g[k], t[name].grad.numpy(), rtol=0, atol=1e-12)
