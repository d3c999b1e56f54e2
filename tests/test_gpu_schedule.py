"""The layer sequences of the workloads: the cyclic window schedule (windows
16/32/64, shift on the middle layer) with forward and backward per layer, and
the 12-layer 96x96-window inference that computes Qp/Kp once and reuses them
for every window and layer.  End to end: position tokens from the GPU kernel,
checked against the oracle's fp64 tokens and attention."""
import numpy as np
import pytest
import torch

import oracle as O
import rib_inputs as I
import windowed_attention_implicit_b200 as R
from windowed_attention_implicit_b200.schedule import LayerSpec, RIBLayerStack
from tests.rib_testlib import assert_all, bf16_round, check_close, to_np

pytestmark = pytest.mark.gpu


def test_cyclic_window_schedule_fwd_bwd(bwd_kernel):
    w = I.get_workload("cyclic", batch=1, heads=2)
    layers, inputs = [], []
    for l in range(w.layers):
        inp = I.make_layer_inputs(w, l, strong=True)
        mlp = R.PositionMLP.from_params(inp["freqs"], inp["mlp_q"], inp["mlp_k"], w.heads, w.rank)
        layers.append(LayerSpec(inp["window"], inp["shift"], mlp))
        inputs.append(inp)
    stack = RIBLayerStack(layers)
    qkvs = [inp["qkv"].cuda() for inp in inputs]
    states = stack.forward(qkvs)
    grads = stack.backward(qkvs, states, [inp["dout"].cuda() for inp in inputs], mlp_grads=False)
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    assert len(stack.cache) == 3            # one Qp/Kp set per geometry
    checks = []
    for l, (spec, inp, st, g) in enumerate(zip(layers, inputs, states, grads)):
        # the attention consumes bf16 copies of the tokens: the oracle takes
        # the bf16 rounding of its own fp64 tokens
        qp, kp = O.pos_tokens(inp["freqs"], inp["mlp_q"], inp["mlp_k"], spec.window, w.heads,
                              w.rank)
        qp, kp = bf16_round(qp), bf16_round(kp)
        ro, rl = O.attn_fwd(inp["qkv"], spec.window, spec.shift, qp, kp)
        checks.append(check_close(to_np(st.out), ro, f"layer {l} (M={spec.window}) out"))
        checks.append(check_close(to_np(st.lse), rl, f"layer {l} lse"))
        dq, dqp, dkp = O.attn_bwd(inp["qkv"], inp["dout"], spec.window, spec.shift, qp, kp)
        checks.append(check_close(to_np(g["dqkv"]), dq, f"layer {l} dqkv"))
        checks.append(check_close(to_np(g["dqp"]), dqp, f"layer {l} dQp", normalize=True))
        checks.append(check_close(to_np(g["dkp"]), dkp, f"layer {l} dKp", normalize=True))
    assert_all(checks)


def test_twelve_layer_inference_reuses_position_tokens():
    w = I.get_workload("w96infer")
    inp0 = I.make_layer_inputs(w, 0, strong=True)
    mlp = R.PositionMLP.from_params(inp0["freqs"], inp0["mlp_q"], inp0["mlp_k"], w.heads, w.rank)
    stack = RIBLayerStack([LayerSpec(w.windows[l], w.shifts[l], mlp) for l in range(w.layers)])
    qkvs = [I.make_layer_inputs(w, l, strong=True, with_dout=False)["qkv"].cuda()
            for l in range(w.layers)]
    R.rib_trace_enable(True)
    states = stack.forward(qkvs)
    torch.cuda.synchronize()
    kern = R.rib_trace_collect()
    R.rib_trace_enable(False)
    assert R.rib_last_status()[0] == 0
    assert len(stack.cache) == 1 and kern["pos_tokens_kernel"][0] == 1     # computed once
    assert kern["attn_fwd_kernel"][0] == 12
    M = w.windows[0]
    qp, kp = O.pos_tokens(inp0["freqs"], inp0["mlp_q"], inp0["mlp_k"], M, w.heads, w.rank)
    qp, kp = bf16_round(qp).double().numpy(), bf16_round(kp).double().numpy()
    tau = O.default_scale(32, w.rank)
    rng = np.random.default_rng(9)
    nWx = w.width // M
    checks = []
    for l in (0, 1, 11):
        s = w.shifts[l]
        qkv_host = qkvs[l].cpu()
        out = to_np(states[l].out)
        for (win, h) in ((0, 0), (23, 5), (10, 2)):
            rows = np.sort(rng.choice(M * M, 64, replace=False))
            qc, kc, v, qpf, kpf = O.gather_unit(qkv_host, qp, kp, M, s, 0, win, h)
            ro, _ = O.attention_unit_rows(qc, kc, v, qpf, kpf, tau, rows=rows)
            wy, wx = win // nWx, win % nWx
            y = (wy * M + rows // M + s) % w.height
            x = (wx * M + rows % M + s) % w.width
            checks.append(check_close(out[0, y, x, h], ro, f"layer {l} window {win} head {h}"))
    assert_all(checks)
