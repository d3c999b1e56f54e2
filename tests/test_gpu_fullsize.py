"""Parity at the benchmark's full size and launch configuration: the 96x96-
window training workload (B=4, 192x192 map, 6 heads, shift 48).

Forward: sampled query rows of sampled units, computed row by row by the
oracle.  Backward: the upstream gradient is zero outside two sampled units,
so every gradient (dqkv over the whole map, dQp, dKp, the MLP weight grads)
has an exact oracle value from those two units alone.
"""
import numpy as np
import pytest
import torch

import oracle as O
import rib_inputs as I
import windowed_attention_implicit_b200 as R
from tests.rib_testlib import assert_all, bf16_round, check_close, mlp_grad_checks, to_np

pytestmark = pytest.mark.gpu

W96 = I.get_workload("w96train")


def _setup(strong):
    w = W96
    inp = I.make_layer_inputs(w, 0, strong=strong)
    M, s = w.windows[0], w.shifts[0]
    qp, kp = O.pos_tokens(inp["freqs"], inp["mlp_q"], inp["mlp_k"], M, w.heads, w.rank)
    return w, inp, M, s, bf16_round(qp), bf16_round(kp)


@pytest.mark.parametrize("strong", [False, True])
def test_fullsize_fwd_sampled_rows(strong):
    w, inp, M, s, q16, k16 = _setup(strong)
    qkv = inp["qkv"]
    out, lse = R.rib_window_attn_fwd(qkv.cuda(), M, s, q16.cuda(), k16.cuda())
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    out, lse = to_np(out), to_np(lse)
    rng = np.random.default_rng(5)
    nWx = w.width // M
    checks = []
    tau = O.default_scale(32, w.rank)
    for (b, win, h) in [(0, 0, 0), (3, 3, 5), (1, 2, 3)]:
        rows = np.sort(rng.choice(M * M, 96, replace=False))
        qc, kc, v, qpf, kpf = O.gather_unit(qkv, q16, k16, M, s, b, win, h)
        ro, rl = O.attention_unit_rows(qc, kc, v, qpf, kpf, tau, rows=rows)
        wy, wx = win // nWx, win % nWx
        i, j = rows // M, rows % M
        y = (wy * M + i + s) % w.height
        x = (wx * M + j + s) % w.width
        checks.append(check_close(out[b, y, x, h], ro, f"out unit {(b, win, h)}"))
        checks.append(check_close(lse[b, h, y, x], rl, f"lse unit {(b, win, h)}"))
    assert_all(checks)


@pytest.mark.parametrize("strong", [False, True])
def test_fullsize_bwd_two_units(strong):
    w, inp, M, s, q16, k16 = _setup(strong)
    keep = {(0, 1, 2), (0, 2, 5)}                # (batch, window, head)
    dout = inp["dout"].clone()
    dw = O.window_partition(dout.float().numpy(), M, s)
    mask = np.zeros(dw.shape[:2] + dw.shape[3:4], dtype=bool)   # [B, nW, heads]
    for b, win, h in keep:
        mask[b, win, h] = True
    dw = dw * mask[:, :, None, :, None]
    dout = torch.from_numpy(O.window_reverse(dw, M, s, w.height, w.width)).to(torch.bfloat16)

    mlp = R.PositionMLP.from_params(inp["freqs"], inp["mlp_q"], inp["mlp_k"], w.heads, w.rank)
    d_qkv, d_q16, d_k16 = inp["qkv"].cuda(), q16.cuda(), k16.cuda()
    out, lse = R.rib_window_attn_fwd(d_qkv, M, s, d_q16, d_k16)
    g = R.rib_window_attn_bwd(d_qkv, out, dout.cuda(), lse, M, s, d_q16, d_k16, mlp=mlp)
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0

    got = to_np(g["dqkv"])
    assert not np.any(got[1:]), "batch entries without upstream gradient must get zero"
    rq, rqp, rkp = O.attn_bwd(inp["qkv"][0:1], dout[0:1], M, s, q16, k16, units=keep)
    checks = [check_close(got[0:1, :, :, k], rq[:, :, :, k], name)
              for k, name in enumerate(("dQc", "dKc", "dV"))]
    checks.append(check_close(to_np(g["dqp"]), rqp, "dQp", normalize=True))
    checks.append(check_close(to_np(g["dkp"]), rkp, "dKp", normalize=True))
    gq, gk = O.pos_tokens_backward(inp["freqs"], inp["mlp_q"], inp["mlp_k"], M, rqp, rkp)
    checks += mlp_grad_checks(g["dmlp"], gq, gk)
    assert_all(checks)


def test_fullsize_key_gradients_sum_to_zero_in_every_unit():
    """Property that holds at any size: rows of dS sum to zero, so in every
    unit the keys' gradients dKc (and dKp) sum to zero.  Checked over all 96
    units of the full workload with its real upstream gradient; the bound is
    1% of the summed magnitude (bf16 rounding is 0.2% per element)."""
    w, inp, M, s, q16, k16 = _setup(True)
    d_qkv = inp["qkv"].cuda()
    out, lse = R.rib_window_attn_fwd(d_qkv, M, s, q16.cuda(), k16.cuda())
    g = R.rib_window_attn_bwd(d_qkv, out, inp["dout"].cuda(), lse, M, s, q16.cuda(), k16.cuda())
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    dk = O.window_partition(to_np(g["dqkv"])[:, :, :, 1], M, s)      # [B, nW, N, heads, d]
    tot = dk.sum(axis=2)
    mass = np.abs(dk).sum(axis=2)
    worst = float((np.abs(tot) / np.maximum(mass, 1e-30)).max())
    print(f"max |sum_k dKc| / sum_k |dKc| over units and channels: {worst:.3e}")
    assert worst <= 1e-2
