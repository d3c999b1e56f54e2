"""Planted mistakes in the CLA oracle must be caught by its pins: each case
monkeypatches one oracle function with a plausible bug and at least one pin
of tests/test_cla_oracle.py must then fail."""
import numpy as np
import pytest

import oracle as O
from oracle import cla_oracle as C
import tests.test_cla_oracle as P

_orig_dw = C.dw_conv3x3


def _dw_convolution_not_correlation(x, w_dw, b_dw):
    return _orig_dw(x, np.asarray(w_dw)[:, ::-1, ::-1], b_dw)


def _dw_no_bias(x, w_dw, b_dw):
    return _orig_dw(x, w_dw, np.zeros_like(np.asarray(b_dw, dtype=np.float64)))


def _pw_transposed(y, w_pw, b_pw):
    return C._f64(y) @ C._f64(w_pw) + C._f64(b_pw)


def _sigmoid_sign(z):
    return 1.0 / (1.0 + np.exp(C._f64(z)))


_orig_bwd = C.cla_backward


def _bwd_missing_gate_derivative(x, w_dw, b_dw, w_pw, b_pw, o, d_out):
    g = _orig_bwd(x, w_dw, b_dw, w_pw, b_pw, o, d_out)
    gate = C.cla_gate(x, w_dw, b_dw, w_pw, b_pw)
    g["db_pw"] = (C._f64(d_out).reshape(gate.shape) * C._f64(o).reshape(gate.shape)).sum(axis=(0, 1, 2))
    return g


def _bwd_dx_without_flip(x, w_dw, b_dw, w_pw, b_pw, o, d_out):
    g = _orig_bwd(x, w_dw, b_dw, w_pw, b_pw, o, d_out)
    g2 = _orig_bwd(x, np.asarray(w_dw)[:, ::-1, ::-1], b_dw, w_pw, b_pw, o, d_out)
    g["dx"] = g2["dx"]
    return g


CASES = [
    ("dw_conv3x3", _dw_convolution_not_correlation, ["test_dw_conv_matches_torch_grouped_conv2d_fp64",
                                                     "test_interior_impulse_spreads_the_kernel_by_cross_correlation"]),
    ("dw_conv3x3", _dw_no_bias, ["test_dw_conv_matches_torch_grouped_conv2d_fp64"]),
    ("pw_conv", _pw_transposed, ["test_pw_conv_matches_torch_1x1_conv2d_fp64"]),
    ("sigmoid", _sigmoid_sign, ["test_sigmoid_closed_forms", "test_zero_pointwise_weight_gives_constant_gate"]),
    ("cla_backward", _bwd_missing_gate_derivative, ["test_backward_matches_torch_autograd_fp64"]),
    ("cla_backward", _bwd_dx_without_flip, ["test_backward_matches_torch_autograd_fp64"]),
]


@pytest.mark.parametrize("fn,bad,pins", CASES, ids=[c[1].__name__ for c in CASES])
def test_planted_mistake_is_caught(monkeypatch, fn, bad, pins):
    monkeypatch.setattr(C, fn, bad)
    monkeypatch.setattr(O, fn, bad)
    caught = 0
    for name in pins:
        try:
            getattr(P, name)()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin caught the planted mistake in {fn}"
