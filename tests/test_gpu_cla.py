"""GPU parity of the convolutional local attention gate (rib_cla_gate) and of
the gated forward (rib_window_attn_fwd_cla) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle as O
import rib_inputs as I
import windowed_attention_implicit_b200 as R
from tests.rib_testlib import Case, assert_all, assert_close, check_close, to_np

pytestmark = pytest.mark.gpu


def _gate(B, H, W, C, seed):
    x = I.make_features(B, H, W, C, seed)
    p = I.make_cla(C, seed)
    cla = R.ClaGate.from_params(p.w_dw, p.b_dw, p.w_pw, p.b_pw)
    return x, p, cla


@pytest.mark.parametrize("B,H,W,C", [
    (1, 8, 16, 32),       # one tile: every pixel touches the zero padding
    (1, 24, 48, 96),      # tiny workload's width (3 heads), partial 64-channel group
    (2, 32, 32, 192),     # six heads, several tiles per image, two images
    (1, 16, 32, 160),     # five heads: a partial 64-channel halo box
])
def test_cla_gate_parity(B, H, W, C):
    x, p, cla = _gate(B, H, W, C, seed=C + H)
    g = R.rib_cla_gate(x.cuda(), cla)
    torch.cuda.synchronize()
    code, site = R.rib_last_status()
    assert code == 0, (code, site)
    ref = O.cla_gate(x, p.w_dw, p.b_dw, p.w_pw, p.b_pw)
    assert_close(to_np(g), ref, f"gate B={B} {H}x{W} C={C}")


def test_cla_gate_full_size_map():
    """The 96x96-window training map: B=4, 192x192, C=192 (all 1152 tiles,
    the persistent grid's every CTA), compared on every pixel."""
    x, p, cla = _gate(4, 192, 192, 192, seed=3)
    g = R.rib_cla_gate(x.cuda(), cla)
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    ref = O.cla_gate(x, p.w_dw, p.b_dw, p.w_pw, p.b_pw)
    assert_close(to_np(g), ref, "gate 4x192x192x192")


@pytest.mark.parametrize("args", [
    dict(B=1, H=64, W=64, heads=3, M=16, s=0),
    dict(B=2, H=64, W=96, heads=6, M=32, s=16),
])
def test_attn_fwd_cla_parity(args):
    c = Case(seed=11, **args)
    C = c.heads * 32
    x, p, cla = _gate(c.B, c.H, c.W, C, seed=5)
    d = c.device()
    gate = R.rib_cla_gate(x.cuda(), cla)
    out, out_g, lse = R.rib_window_attn_fwd_cla(d["qkv"], c.M, c.s, gate, d["qp16"], d["kp16"])
    out0, lse0 = R.rib_window_attn_fwd(d["qkv"], c.M, c.s, d["qp16"], d["kp16"])
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    # the ungated output and lse are the plain forward's, bit for bit
    assert torch.equal(out, out0) and torch.equal(lse, lse0)
    ro, rl = c.oracle_fwd()
    rg = O.cla_gate(x, p.w_dw, p.b_dw, p.w_pw, p.b_pw)
    assert_close(to_np(out_g), O.cla_apply(ro, rg), "gated output")
    assert_close(to_np(out), ro, "ungated output")


def test_cla_gate_rejects_bad_shapes():
    x = torch.zeros((1, 8, 16, 48), device="cuda", dtype=torch.bfloat16)
    p = I.make_cla(48, 1)
    cla = R.ClaGate.from_params(p.w_dw, p.b_dw, p.w_pw, p.b_pw)
    with pytest.raises(R.RibError):
        R.rib_cla_gate(x, cla)                      # C % 32 != 0
    x = torch.zeros((1, 12, 16, 64), device="cuda", dtype=torch.bfloat16)
    p = I.make_cla(64, 1)
    cla = R.ClaGate.from_params(p.w_dw, p.b_dw, p.w_pw, p.b_pw)
    with pytest.raises(R.RibError):
        R.rib_cla_gate(x, cla)                      # H % 8 != 0
    x = torch.zeros((1, 8, 16, 256), device="cuda", dtype=torch.bfloat16)
    p = I.make_cla(256, 1)
    cla = R.ClaGate.from_params(p.w_dw, p.b_dw, p.w_pw, p.b_pw)
    with pytest.raises(R.RibError):
        R.rib_cla_gate(x, cla)                      # C > 192: no room for the buffers


def _cla_bwd_case(B, H, W, C, seed):
    x, p, cla = _gate(B, H, W, C, seed)
    o = I.make_features(B, H, W, C, seed + 100)          # an ungated output O
    dout_g = I.make_features(B, H, W, C, seed + 200)     # dO'
    xd = x.cuda()
    gate = R.rib_cla_gate(xd, cla)
    g = R.rib_cla_bwd(xd, cla, gate, o.cuda(), dout_g.cuda())
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    ref = O.cla_backward(x, p.w_dw, p.b_dw, p.w_pw, p.b_pw, o, dout_g)
    # dO = dO' * G has the magnitude of the upstream gradient (up to ~5 for
    # N(0,1) draws over 28 M elements), where one bf16 half-ulp is 0.016:
    # measured, like the sums below, against max(1, max|ref|)
    checks = [check_close(to_np(g["dout"]), ref["d_o"], "dO", normalize=True),
              check_close(to_np(g["dx"]), ref["dx"], "dx")]
    # sums over every pixel: measured against their magnitude (bf16 operands)
    for k in ("dw_pw", "db_pw", "dw_dw", "db_dw"):
        checks.append(check_close(to_np(g[k]), ref[k], k, normalize=True))
    assert_all(checks)
    return g


@pytest.mark.parametrize("B,H,W,C", [
    (1, 8, 16, 32),       # one tile, every pixel at the border
    (1, 16, 32, 96),      # three heads, a partial 64-channel group
    (2, 32, 48, 192),     # six heads (two point-wise accumulators), several tiles
    (1, 16, 32, 160),     # five heads: a partial last 64-channel chunk and two M blocks
])
def test_cla_bwd_parity(B, H, W, C):
    _cla_bwd_case(B, H, W, C, seed=C + 7)


def test_cla_bwd_full_size_and_deterministic():
    """The w96train map (1152 tiles, every CTA of the persistent grids), and
    bit-identical weight gradients on a second call (fixed-order sums)."""
    g1 = _cla_bwd_case(4, 192, 192, 192, seed=3)
    x, p, cla = _gate(4, 192, 192, 192, 3)
    o = I.make_features(4, 192, 192, 192, 103).cuda()
    dout_g = I.make_features(4, 192, 192, 192, 203).cuda()
    xd = x.cuda()
    g2 = R.rib_cla_bwd(xd, cla, R.rib_cla_gate(xd, cla), o, dout_g)
    torch.cuda.synchronize()
    for k in ("dw_pw", "db_pw", "dw_dw", "db_dw", "dx", "dout"):
        assert torch.equal(g1[k], g2[k]), k


def test_training_layer_with_cla_matches_oracle_composition():
    """One training layer through the library's composed path, gate ->
    gated forward -> CLA backward -> attention backward (fed the CLA
    backward's dO), against the same composition of fp64 oracle functions."""
    c = Case(1, 64, 64, 2, 32, 16, seed=21)
    C = c.heads * 32
    x, p, cla = _gate(c.B, c.H, c.W, C, seed=9)
    dout_g = I.make_features(c.B, c.H, c.W, C, 909)          # dO' of the gated output
    d = c.device()
    xd = x.cuda()
    gate = R.rib_cla_gate(xd, cla)
    out, out_g, lse = R.rib_window_attn_fwd_cla(d["qkv"], c.M, c.s, gate, d["qp16"], d["kp16"])
    g = R.rib_cla_bwd(xd, cla, gate, out, dout_g.cuda())
    ga = R.rib_window_attn_bwd(d["qkv"], out, g["dout"], lse, c.M, c.s, d["qp16"], d["kp16"])
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    ro, _ = c.oracle_fwd()
    rg = O.cla_gate(x, p.w_dw, p.b_dw, p.w_pw, p.b_pw)
    rc = O.cla_backward(x, p.w_dw, p.b_dw, p.w_pw, p.b_pw, ro, dout_g)
    d_o = rc["d_o"].reshape(c.B, c.H, c.W, c.heads, 32)
    rdq, rdqp, rdkp = O.attn_bwd(c.qkv, d_o, c.M, c.s, c.qp16, c.kp16, c.scale)
    checks = [check_close(to_np(out_g), O.cla_apply(ro, rg), "gated output"),
              check_close(to_np(g["dx"]), rc["dx"], "dx"),
              check_close(to_np(ga["dqkv"]), rdq, "dqkv"),
              check_close(to_np(ga["dqp"]), rdqp, "dqp", normalize=True),
              check_close(to_np(ga["dkp"]), rdkp, "dkp", normalize=True)]
    for k in ("dw_pw", "db_pw", "dw_dw", "db_dw"):
        checks.append(check_close(to_np(g[k]), rc[k], k, normalize=True))
    assert_all(checks)
