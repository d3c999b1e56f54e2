"""GPU edge cases: empty batches, large logits (lazy rescale of the running
maximum, the FMA-pipe exponential's low clamp) and the largest windows."""
import numpy as np
import pytest
import torch

import oracle as O
import rib_inputs as I
import windowed_attention_implicit_b200 as R
from tests.rib_testlib import Case, assert_all, check_close, to_np

pytestmark = pytest.mark.gpu


def test_empty_batch_forward_and_backward():
    """B = 0: nothing to compute; the backward's sums over batch entries and
    windows (dQp, dKp, the position-MLP gradients) are empty sums, zero."""
    heads, M, r, F, hid = 2, 32, 16, 16, 64
    dev = "cuda"
    qkv = torch.empty((0, 64, 64, 3, heads, 32), device=dev, dtype=torch.bfloat16)
    mq = I.make_mlp(F, hid, heads, r, 1, 0, strong=True)
    mk = I.make_mlp(F, hid, heads, r, 1, 1, strong=True)
    mlp = R.PositionMLP.from_params(I.default_freqs(F), mq, mk, heads, r)
    _, _, q16, k16 = R.rib_pos_tokens(mlp, M)
    out, lse = R.rib_window_attn_fwd(qkv, M, 0, q16, k16)
    assert out.shape[0] == 0 and lse.shape[0] == 0
    nan = lambda t: torch.full_like(t, float("nan"))
    dqp, dkp = nan(q16.float()), nan(k16.float())
    dmlp = R.PositionMLPGrad(*[nan(t) for t in (mlp.q_w1, mlp.q_b1, mlp.q_w2, mlp.q_b2,
                                                mlp.k_w1, mlp.k_b1, mlp.k_w2, mlp.k_b2)])
    g = R.rib_window_attn_bwd(qkv, out, torch.empty_like(out), lse, M, 0, q16, k16, mlp=mlp,
                              dqp=dqp, dkp=dkp, dmlp=dmlp)
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    assert g["dqkv"].shape[0] == 0
    for t in [dqp, dkp] + list(dmlp.tensors().values()):
        assert torch.count_nonzero(t).item() == 0 and not torch.isnan(t).any()
    # the CLA backward likewise zeroes its weight gradients
    p = I.make_cla(64, 2)
    cla = R.ClaGate.from_params(p.w_dw, p.b_dw, p.w_pw, p.b_pw)
    x = torch.empty((0, 16, 32, 64), device=dev, dtype=torch.bfloat16)
    gate = R.rib_cla_gate(x, cla)
    gc = R.rib_cla_bwd(x, cla, gate, torch.empty_like(x), torch.empty_like(x))
    torch.cuda.synchronize()
    for k in ("dw_dw", "db_dw", "dw_pw", "db_pw"):
        assert torch.count_nonzero(gc[k]).item() == 0, k


def test_large_logits_fwd_bwd_parity():
    """qkv ~ N(0, 4^2): scaled logits of std ~13, so the running row maximum
    grows past the lazy-rescale threshold on many key tiles and exponents
    fall far below the FMA-pipe polynomial's clamp.  Outputs and gradients
    grow with the inputs, so errors are measured against max(1, max|ref|)."""
    c = Case(1, 64, 64, 2, 32, 16, seed=13, qkv_std=4.0)
    d = c.device()
    out, lse = R.rib_window_attn_fwd(d["qkv"], c.M, c.s, d["qp16"], d["kp16"])
    g = R.rib_window_attn_bwd(d["qkv"], out, d["dout"], lse, c.M, c.s, d["qp16"], d["kp16"])
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    ro, rl = c.oracle_fwd()
    rdq, rdqp, rdkp = c.oracle_bwd()
    assert np.abs(rl).max() > 50.0      # the case really has large logits
    assert_all([check_close(to_np(out), ro, "out", normalize=True,
                            grown_inputs=True),
                check_close(to_np(lse), rl, "lse", normalize=True,
                            grown_inputs=True),
                check_close(to_np(g["dqkv"]), rdq, "dqkv", normalize=True,
                            grown_inputs=True),
                check_close(to_np(g["dqp"]), rdqp, "dqp", normalize=True,
                            grown_inputs=True),
                check_close(to_np(g["dkp"]), rdkp, "dkp", normalize=True,
                            grown_inputs=True)])


@pytest.mark.parametrize("M,heads", [(128, 2), (256, 1)])
def test_largest_windows(M, heads):
    """The largest windows the library accepts: forward on sampled query rows
    of every unit against the oracle; backward through its invariant that
    every unit's key gradients sum to zero (rows of dS sum to zero)."""
    c = Case(1, M, M, heads, M, 8, seed=31)
    d = c.device()
    out, lse = R.rib_window_attn_fwd(d["qkv"], M, c.s, d["qp16"], d["kp16"])
    g = R.rib_window_attn_bwd(d["qkv"], out, d["dout"], lse, M, c.s, d["qp16"], d["kp16"])
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    out, lse, dqkv, dkp = to_np(out), to_np(lse), to_np(g["dqkv"]), to_np(g["dkp"])
    rng = np.random.default_rng(M)
    checks = []
    for h in range(heads):
        rows = np.sort(rng.choice(M * M, 64, replace=False))
        qc, kc, v, qpf, kpf = O.gather_unit(c.qkv, c.qp16, c.kp16, M, c.s, 0, 0, h)
        ro, rl = O.attention_unit_rows(qc, kc, v, qpf, kpf, c.scale, rows=rows)
        y = (rows // M + c.s) % M
        x = (rows % M + c.s) % M
        checks.append(check_close(out[0, y, x, h], ro, f"out M={M} head {h}"))
        checks.append(check_close(lse[0, h, y, x], rl, f"lse M={M} head {h}"))
        # one window per image here, so dKc over the map and dKp are the unit's
        dk = dqkv[0, :, :, 1, h, :].reshape(-1, 32)
        # (bound as for the full-size workload: 1 % of the summed magnitude
        # per channel; bf16 rounding is 0.2 % per element)
        for name, grad in (("dKc", dk), ("dKp", dkp[h].reshape(-1, 16))):
            worst = float((np.abs(grad.sum(axis=0)) / np.maximum(np.abs(grad).sum(axis=0), 1e-30)).max())
            assert worst <= 1e-2, f"{name} M={M} head {h}: {worst:.3e}"
    assert_all(checks)
