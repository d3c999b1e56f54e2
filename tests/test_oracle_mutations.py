"""Planted mistakes in the oracle must be caught by its pins.

Each case monkeypatches one oracle function with a plausible bug (dropped
term, wrong sign, transposed operand, swapped index) and runs the pin tests
that should catch it; at least one of them must fail.
"""
import inspect

import numpy as np
import pytest

import oracle as O
from oracle import rib_oracle as R
import tests.test_oracle_pins as P


def _masked(sc, allowed):
    return sc if allowed is None else np.where(allowed, sc, -np.inf)


def _scores_bias_sign(qc, kc, qp, kp, scale, allowed=None):
    return _masked(scale * (R._f64(qc) @ R._f64(kc).T - R._f64(qp) @ R._f64(kp).T), allowed)


def _scores_no_bias(qc, kc, qp, kp, scale, allowed=None):
    return _masked(scale * (R._f64(qc) @ R._f64(kc).T), allowed)


def _fourier_swapped(y, x, freqs):
    w = R._f64(freqs).reshape(1, -1)
    ax = np.asarray(x, dtype=np.float64).reshape(-1, 1) * w
    ay = np.asarray(y, dtype=np.float64).reshape(-1, 1) * w
    return np.concatenate([np.sin(ay), np.cos(ay), np.sin(ax), np.cos(ax)], 1)


def _coords_no_endpoint(M):
    lin = -1.0 + 2.0 * np.arange(M, dtype=np.float64) / M
    return np.repeat(lin, M), np.tile(lin, M)


def _gelu_tanh(z):
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1 + np.tanh(np.sqrt(2 / np.pi) * (z + 0.044715 * z ** 3)))


def _partition_wrong_roll(x, M, s):
    return _orig_partition(np.roll(np.asarray(x), shift=(s, s), axis=(1, 2)), M, 0)


_orig_partition = R.window_partition


def _bwd_missing_rowsum(qc, kc, v, qp, kp, scale, dout, labels=None):
    qc, kc, v, qp, kp, do = map(R._f64, (qc, kc, v, qp, kp, dout))
    s = R.unit_scores(qc, kc, qp, kp, scale, R._allowed(labels, 0, qc.shape[0]))
    p, _ = R._softmax_rows(s)
    dp = do @ v.T
    ds = p * dp
    return (scale * ds @ kc, scale * ds.T @ qc, p.T @ do, scale * ds @ kp,
            scale * ds.T @ qp)


def _bwd_dk_transposed(qc, kc, v, qp, kp, scale, dout, labels=None):
    g = list(_orig_unit_bwd(qc, kc, v, qp, kp, scale, dout, labels=labels))
    g[4] = scale * 0 + g[3][: g[4].shape[0]]          # dKp taken from dQp
    return tuple(g)


_orig_unit_bwd = R.attention_unit_backward


def _mlp_bwd_no_gelu_grad(gamma, w1, b1, w2, b2, d_out):
    a, h, _ = R.mlp_forward(gamma, w1, b1, w2, b2)
    g = R._f64(d_out)
    dh = g @ R._f64(w2)
    return dh.T @ gamma, dh.sum(0), g.T @ h, g.sum(0)


def _gather_wrong_head_pos(qkv, qp, kp, M, s, b, w, h):
    g = list(_orig_gather(qkv, qp, kp, M, s, b, w, h))
    g[3] = R._f64(qp)[0].reshape(M * M, -1)          # Qp of head 0 for every head
    return tuple(g)


def _gather_wrong_batch(qkv, qp, kp, M, s, b, w, h):
    return _orig_gather(qkv, qp, kp, M, s, 0, w, h)   # batch entry ignored


def _gather_k_v_swapped(qkv, qp, kp, M, s, b, w, h):
    qc, kc, v, qpf, kpf = _orig_gather(qkv, qp, kp, M, s, b, w, h)
    return qc, v, kc, qpf, kpf


_orig_gather = R.gather_unit


def _allowed_ignores_rows(labels, r0, r1, rows=None):
    return _orig_allowed(labels, r0, r1)              # labels of rows 0.. instead of `rows`


_orig_allowed = R._allowed


def _rows_positional_unsliced(qc, kc, v, qp, kp, scale, rows=None, labels=None):
    qc, kc, v, qp, kp = map(R._f64, (qc, kc, v, qp, kp))
    if rows is not None:
        qc = qc[rows]                                 # Qp left in token order
        qp = qp[: len(rows)]
    n = qc.shape[0]
    out, lse = np.empty((n, v.shape[1])), np.empty(n)
    for r0 in range(0, n, R._ROW_BLOCK):
        r1 = min(n, r0 + R._ROW_BLOCK)
        sc = R.unit_scores(qc[r0:r1], kc, qp[r0:r1], kp, scale, R._allowed(labels, r0, r1, rows))
        p, lse[r0:r1] = R._softmax_rows(sc)
        out[r0:r1] = p @ v
    return out, lse


MUTATIONS = [
    ("unit_scores", _scores_bias_sign,
     [P.test_golden_closed_forms, P.test_attention_matches_torch_sdpa_augmented]),
    ("unit_scores", _scores_no_bias,
     [P.test_golden_closed_forms, P.test_concatenated_dot_product_equals_content_plus_bias]),
    ("fourier_features", _fourier_swapped,
     [P.test_fourier_block_order, P.test_pos_tokens_torch_composition]),
    ("window_coords", _coords_no_endpoint,
     [P.test_coords_closed_form_m3, P.test_coords_corners_and_spacing]),
    ("gelu", _gelu_tanh,
     [P.test_gelu_textbook_values, P.test_gelu_matches_torch_exact_gelu]),
    ("window_partition", _partition_wrong_roll,
     [P.test_partition_matches_modular_index_and_inverts,
      P.test_full_map_against_per_pixel_brute_force]),
    ("attention_unit_backward", _bwd_missing_rowsum,
     [P.test_attn_bwd_finite_differences, P.test_attn_bwd_matches_torch_autograd]),
    ("attention_unit_backward", _bwd_dk_transposed,
     [P.test_attn_bwd_matches_torch_autograd]),
    ("mlp_backward", _mlp_bwd_no_gelu_grad,
     [P.test_mlp_backward_finite_differences, P.test_pos_tokens_backward_finite_differences]),
    ("gather_unit", _gather_wrong_head_pos,
     [P.test_gather_unit_matches_pixel_index, P.test_gather_unit_then_attention_is_the_map_output]),
    ("gather_unit", _gather_wrong_batch,
     [P.test_gather_unit_matches_pixel_index, P.test_gather_unit_then_attention_is_the_map_output]),
    ("gather_unit", _gather_k_v_swapped,
     [P.test_gather_unit_matches_pixel_index]),
    ("_allowed", _allowed_ignores_rows,
     [P.test_attention_unit_rows_matches_per_row_brute_force]),
    ("attention_unit_rows", _rows_positional_unsliced,
     [P.test_attention_unit_rows_matches_per_row_brute_force]),
]

_PARAMS = {
    P.test_coords_corners_and_spacing: {"M": 5},
    P.test_concatenated_dot_product_equals_content_plus_bias: {"r": 3},
    P.test_attention_matches_torch_sdpa_augmented: {"r": 16},
    P.test_partition_matches_modular_index_and_inverts: {"M": 4, "s": 3},
    P.test_gather_unit_matches_pixel_index: {"M": 2, "s": 1, "b": 1, "w": 5, "h": 2},
    P.test_attention_unit_rows_matches_per_row_brute_force: {"masked": True},
}


@pytest.mark.parametrize("name,bad,pins", MUTATIONS,
                         ids=[f"{m[0]}:{m[1].__name__}" for m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, name, bad, pins):
    monkeypatch.setattr(R, name, bad)
    if hasattr(O, name):
        monkeypatch.setattr(O, name, bad)
    caught = 0
    for pin in pins:
        kw = dict(_PARAMS.get(pin, {}))
        if "monkeypatch" in inspect.signature(pin).parameters:
            kw["monkeypatch"] = monkeypatch
        try:
            pin(**kw)
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake in {name}"


_PIN_FILES = ("test_oracle_pins.py", "test_region_mask_oracle.py", "test_cla_oracle.py")


def test_every_exported_oracle_function_is_called_by_a_pin_file():
    """No exported oracle function goes without a CPU pin: each name appears as
    a call in at least one of the pin files (closed forms, brute force,
    library routines, finite differences)."""
    import os
    import re
    here = os.path.dirname(__file__)
    text = "".join(open(os.path.join(here, f)).read() for f in _PIN_FILES)
    missing = [n for n in O.__all__ if not re.search(r"\bO\.%s\(" % n, text)]
    assert not missing, missing
