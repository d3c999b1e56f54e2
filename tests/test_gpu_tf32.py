"""The fp32 forward on the tf32 tensor cores (rib_window_attn_fwd_tf32)
against the fp64 oracle fed the same unrounded fp32 features and fp32
position tokens.  The tiny workload is stated in fp32; the other cases
cover several tiles per unit, a shift, rank 0 and the largest window of
the workloads.

Two bounds apply: the stated one for the attention outputs (max 2e-2,
mean 2e-3), and, element by element, the first-order error bound that
follows from tf32's 10-bit mantissa (tests/rib_testlib.tf32_error_bounds).
A third test checks that the tf32 path is clearly closer to the exact
result than the bf16 path on the same fp32 inputs."""
import numpy as np
import pytest
import torch

import oracle as O
import rib_inputs as I
import windowed_attention_implicit_b200 as R
from tests.rib_testlib import (assert_all, check_close, check_within_bound, tf32_error_bounds,
                               to_np)

pytestmark = pytest.mark.gpu

CASES = [
    # B, H, W, heads, M, s, rank, hidden, strong
    (1, 64, 64, 3, 16, 0, 16, 64, False),    # the tiny workload, its own weights
    (1, 64, 64, 3, 16, 0, 16, 64, True),     # strong positional bias
    (1, 64, 64, 2, 32, 16, 16, 128, True),   # shifted, 8 tiles per unit
    (2, 32, 48, 2, 16, 8, 16, 64, True),     # H != W, shift of one box
    (1, 64, 64, 2, 32, 0, 0, 64, True),      # rank 0: plain windowed attention
    (1, 96, 96, 1, 96, 48, 16, 128, True),   # a 96x96 window: 72 key tiles
]


def _ids(c):
    return "B{}H{}W{}h{}M{}s{}r{}{}".format(*c[:7], "S" if c[8] else "")


def _fp32_tokens(freqs, mq, mk, M, heads, rank):
    qp, kp = O.pos_tokens(freqs, mq, mk, M, heads, rank)
    return (torch.from_numpy(qp).to(torch.float32), torch.from_numpy(kp).to(torch.float32))


@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_tf32_fwd_parity(case):
    B, H, W, heads, M, s, rank, hid, strong = case
    F = 16
    qkv = I.make_qkv(B, H, W, heads, 32, seed=21, dtype=torch.float32)
    freqs = I.default_freqs(F)
    r = max(rank, 1)
    mq = I.make_mlp(F, hid, heads, r, 21, 0, strong=strong)
    mk = I.make_mlp(F, hid, heads, r, 21, 1, strong=strong)
    if rank:
        qp, kp = _fp32_tokens(freqs, mq, mk, M, heads, rank)
    else:
        qp = kp = torch.zeros((heads, M, M, 0), dtype=torch.float32)
    out, lse = R.rib_window_attn_fwd_tf32(qkv.cuda(), M, s, qp.cuda() if rank else None,
                                          kp.cuda() if rank else None, rank=rank)
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    assert out.dtype == torch.float32
    tau = O.default_scale(32, rank)
    ro, rl = O.attn_fwd(qkv, M, s, qp, kp, tau)
    ob, lb = tf32_error_bounds(qkv, qp, kp, M, s, tau)
    assert_all([check_close(to_np(out), ro, "out"), check_close(to_np(lse), rl, "lse"),
                check_within_bound(to_np(out), ro, ob, "out"),
                check_within_bound(to_np(lse), rl, lb, "lse")])


def test_tf32_tiny_workload_end_to_end():
    """The tiny workload as stated (fp32, its own N(0, 0.02) weights): GPU
    position tokens in fp32 feed the tf32 forward; the oracle computes its
    own tokens in fp64."""
    w = I.get_workload("tiny")
    inp = I.make_layer_inputs(w, 0, qkv_dtype=torch.float32)
    M, s = w.windows[0], w.shifts[0]
    mlp = R.PositionMLP.from_params(inp["freqs"], inp["mlp_q"], inp["mlp_k"], w.heads, w.rank)
    qp, kp, _, _ = R.rib_pos_tokens(mlp, M)
    out, lse = R.rib_window_attn_fwd_tf32(inp["qkv"].cuda(), M, s, qp, kp)
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    rq, rk = O.pos_tokens(inp["freqs"], inp["mlp_q"], inp["mlp_k"], M, w.heads, w.rank)
    tau = O.default_scale(32, w.rank)
    ro, rl = O.attn_fwd(inp["qkv"], M, s, rq, rk, tau)
    # the GPU tokens differ from the fp64 ones by <= 1e-5 relative: far
    # below the tf32 rounding the bound covers
    ob, lb = tf32_error_bounds(inp["qkv"], rq, rk, M, s, tau)
    assert_all([check_close(to_np(out), ro, "out"), check_close(to_np(lse), rl, "lse"),
                check_within_bound(to_np(out), ro, ob, "out"),
                check_within_bound(to_np(lse), rl, lb, "lse")])


def test_tf32_is_closer_to_the_oracle_than_bf16():
    """On the same fp32 features the tf32 path must beat the bf16 path (which
    rounds the features, the tokens and P to bf16) by a clear margin."""
    B, H, W, heads, M, s = 1, 64, 64, 2, 32, 16
    qkv = I.make_qkv(B, H, W, heads, 32, seed=8, dtype=torch.float32)
    freqs = I.default_freqs(16)
    mq = I.make_mlp(16, 64, heads, 16, 8, 0, strong=True)
    mk = I.make_mlp(16, 64, heads, 16, 8, 1, strong=True)
    qp, kp = _fp32_tokens(freqs, mq, mk, M, heads, 16)
    ro, _ = O.attn_fwd(qkv, M, s, qp, kp)
    o32, _ = R.rib_window_attn_fwd_tf32(qkv.cuda(), M, s, qp.cuda(), kp.cuda())
    o16, _ = R.rib_window_attn_fwd(qkv.cuda().to(torch.bfloat16), M, s,
                                   qp.cuda().to(torch.bfloat16), kp.cuda().to(torch.bfloat16))
    torch.cuda.synchronize()
    e32 = np.abs(to_np(o32) - ro).mean()
    e16 = np.abs(to_np(o16) - ro).mean()
    print(f"mean |d|: tf32 {e32:.3e}, bf16 {e16:.3e}")
    assert e32 < e16 / 2


def test_tf32_rejects_bad_arguments():
    q = torch.zeros((1, 32, 32, 3, 1, 32), device="cuda")
    p = torch.zeros((1, 16, 16, 16), device="cuda")
    with pytest.raises(R.RibError):
        R.rib_window_attn_fwd_tf32(q, 16, 4, p, p)            # shift % 8 != 0
    with pytest.raises(ValueError):
        R.rib_window_attn_fwd_tf32(q.to(torch.bfloat16), 16, 0, p, p)
    with pytest.raises(R.RibError):
        R.rib_window_attn_fwd_tf32(q, 16, 0, p[:, :8], p)    # tokens of the wrong size
