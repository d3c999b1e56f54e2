"""Repeatability of the backward.

The key-side gradients (dKc, dV, dKp, the key MLP's weight gradients) come
from sums in a fixed order and must be bit-identical from call to call.  The
query-side ones (dQc, dQp, the query MLP's weight gradients) are folded into
an fp32 accumulator by every key tile of a unit, in an order set by CTA
scheduling: two calls must agree within the parity tolerance, and the test
reports how far apart they are.  The forward (one CTA owns each query tile)
must be bit-identical.
"""
import numpy as np
import pytest
import torch

import rib_inputs as I
import windowed_attention_implicit_b200 as R
from tests.rib_testlib import assert_all, check_close, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,B", [("w32", 2), ("w96train", 4)])
def test_backward_repeatability(name, B, bwd_kernel):
    w = I.get_workload(name)
    inp = I.make_layer_inputs(w, 0, strong=True)
    M, s = w.windows[0], w.shifts[0]
    qkv, dout = inp["qkv"][:B].cuda(), inp["dout"][:B].cuda()
    mlp = R.PositionMLP.from_params(inp["freqs"], inp["mlp_q"], inp["mlp_k"], w.heads, w.rank)
    _, _, q16, k16 = R.rib_pos_tokens(mlp, M)
    runs = []
    for _ in range(3):
        out, lse = R.rib_window_attn_fwd(qkv, M, s, q16, k16)
        g = R.rib_window_attn_bwd(qkv, out, dout, lse, M, s, q16, k16, mlp=mlp)
        torch.cuda.synchronize()
        assert R.rib_last_status()[0] == 0
        runs.append((out.clone(), lse.clone(), g))
    (o0, l0, g0) = runs[0]
    checks = []
    for o, l, g in runs[1:]:
        assert torch.equal(o, o0) and torch.equal(l, l0), "forward must be bit-identical"
        assert torch.equal(g["dqkv"][:, :, :, 1:], g0["dqkv"][:, :, :, 1:]), "dKc / dV"
        assert torch.equal(g["dkp"], g0["dkp"]), "dKp"
        for n in ("k_dw1", "k_db1", "k_dw2", "k_db2"):
            assert torch.equal(getattr(g["dmlp"], n), getattr(g0["dmlp"], n)), n
        checks.append(check_close(to_np(g["dqkv"][:, :, :, 0]), to_np(g0["dqkv"][:, :, :, 0]),
                                  "dQc call to call"))
        checks.append(check_close(to_np(g["dqp"]), to_np(g0["dqp"]), "dQp call to call",
                                  normalize=True))
        for n in ("q_dw1", "q_db1", "q_dw2", "q_db2"):
            a, b = to_np(getattr(g["dmlp"], n)), to_np(getattr(g0["dmlp"], n))
            rel = np.abs(a - b).max() / max(np.abs(b).max(), 1e-30)
            print(f"{n} call to call: rel {rel:.3e}")
            checks.append("" if rel <= 1e-4 else f"{n} rel {rel:.3e}")
        same = torch.equal(g["dqkv"][:, :, :, 0], g0["dqkv"][:, :, :, 0])
        print(f"{name}: dQc bit-identical across calls: {same}")
    assert_all(checks)


def test_backward_dqkv_at_16_byte_offset():
    """dqkv at an address 16- but not 32-byte aligned (the smallest the ABI
    accepts): the dQ write takes its 16-byte store path and the gradients
    match the call with an aligned dqkv (dKc, dV bit-identical; dQc within
    the call-to-call bound of its reduction order)."""
    w = I.get_workload("w32")
    inp = I.make_layer_inputs(w, 0, strong=True)
    M, s = w.windows[0], w.shifts[0]
    qkv, dout = inp["qkv"][:1].cuda(), inp["dout"][:1].cuda()
    mlp = R.PositionMLP.from_params(inp["freqs"], inp["mlp_q"], inp["mlp_k"], w.heads, w.rank)
    _, _, q16, k16 = R.rib_pos_tokens(mlp, M)
    out, lse = R.rib_window_attn_fwd(qkv, M, s, q16, k16)
    g0 = R.rib_window_attn_bwd(qkv, out, dout, lse, M, s, q16, k16)
    buf = torch.empty(qkv.numel() + 64, dtype=torch.bfloat16, device="cuda")
    off = 8 if buf.data_ptr() % 32 == 0 else 24   # 16 bytes past a 32-byte boundary
    dq = buf[off:off + qkv.numel()].view(qkv.shape)
    assert dq.data_ptr() % 32 == 16
    g1 = R.rib_window_attn_bwd(qkv, out, dout, lse, M, s, q16, k16, dqkv=dq,
                               dqp=torch.empty_like(g0["dqp"]), dkp=torch.empty_like(g0["dkp"]))
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    assert torch.equal(g1["dqkv"][:, :, :, 1:], g0["dqkv"][:, :, :, 1:]), "dKc / dV"
    assert_all([check_close(to_np(g1["dqkv"][:, :, :, 0]), to_np(g0["dqkv"][:, :, :, 0]),
                            "dQc, 16-byte-offset dqkv against aligned")])


def _offset_like(t):
    """A tensor shaped like t whose data starts 16 bytes past a 32-byte boundary."""
    n = t.numel()
    buf = torch.empty(n + 64, dtype=t.dtype, device=t.device)
    step = 16 // t.element_size()
    off = step if buf.data_ptr() % 32 == 0 else 3 * step
    v = buf[off:off + n].view(t.shape)
    assert v.data_ptr() % 32 == 16
    return v


def test_forward_outputs_at_16_byte_offset():
    """out and out_gated 16- but not 32-byte aligned: the epilogue takes its
    16-byte store path; the results are bit-identical to aligned outputs."""
    w = I.get_workload("w32")
    inp = I.make_layer_inputs(w, 0, strong=True)
    M, s = w.windows[0], w.shifts[0]
    qkv = inp["qkv"][:1].cuda()
    mlp = R.PositionMLP.from_params(inp["freqs"], inp["mlp_q"], inp["mlp_k"], w.heads, w.rank)
    _, _, q16, k16 = R.rib_pos_tokens(mlp, M)
    o0, l0 = R.rib_window_attn_fwd(qkv, M, s, q16, k16)
    o1 = _offset_like(o0)
    R.rib_window_attn_fwd(qkv, M, s, q16, k16, out=o1, lse=torch.empty_like(l0))
    C = w.heads * w.head_dim
    p = I.make_cla(C, 3)
    cla = R.ClaGate.from_params(p.w_dw, p.b_dw, p.w_pw, p.b_pw)
    x = I.make_features(1, w.height, w.width, C, 3).cuda()
    gate = R.rib_cla_gate(x, cla)
    _, og0, _ = R.rib_window_attn_fwd_cla(qkv, M, s, gate, q16, k16)
    og1 = _offset_like(og0)
    R.rib_window_attn_fwd_cla(qkv, M, s, gate, q16, k16, out=torch.empty_like(o0),
                              out_gated=og1, lse=torch.empty_like(l0))
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    assert torch.equal(o1, o0), "O at a 16-byte offset"
    assert torch.equal(og1, og0), "O * G at a 16-byte offset"
