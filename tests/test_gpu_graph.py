"""The training step captured in a CUDA graph.

Every work entry point only enqueues kernels on the caller's stream (no
synchronous CUDA call, no device allocation: outputs and workspaces are the
caller's tensors), so a whole step - position tokens, forward, backward with
the position-MLP gradients - can be captured once with torch.cuda.graph and
replayed.  The replay must give what the eager calls give (bit-identical
where the sums run in a fixed order; the query-side gradients, reduced in
CTA-scheduling order, within the call-to-call bound), and a replay after the
inputs change in place must follow the new inputs.
"""
import pytest
import torch

import rib_inputs as I
import windowed_attention_implicit_b200 as R
from tests.rib_testlib import assert_all, check_close, to_np

pytestmark = pytest.mark.gpu


def _step_fn(name):
    w = I.get_workload(name)
    inp = I.make_layer_inputs(w, 0, strong=True)
    M, s = w.windows[0], w.shifts[0]
    qkv, dout = inp["qkv"].cuda(), inp["dout"].cuda()
    mlp = R.PositionMLP.from_params(inp["freqs"], inp["mlp_q"], inp["mlp_k"], w.heads, w.rank)
    ws = torch.empty(R.rib_window_attn_bwd_workspace(w.batch, w.height, w.width, w.heads,
                                                     w.head_dim, M, w.rank, mlp),
                     device="cuda", dtype=torch.uint8)

    def step():
        _, _, q16, k16 = R.rib_pos_tokens(mlp, M)
        out, lse = R.rib_window_attn_fwd(qkv, M, s, q16, k16)
        g = R.rib_window_attn_bwd(qkv, out, dout, lse, M, s, q16, k16, mlp=mlp, workspace=ws)
        return out, lse, g

    return w, qkv, step


def _compare(got, ref, tag):
    (o1, l1, g1), (o0, l0, g0) = got, ref
    assert torch.equal(o1, o0) and torch.equal(l1, l0), f"{tag}: forward"
    assert torch.equal(g1["dqkv"][..., 1:, :, :], g0["dqkv"][..., 1:, :, :]), f"{tag}: dKc / dV"
    assert torch.equal(g1["dkp"], g0["dkp"]), f"{tag}: dKp"
    for n in ("k_dw1", "k_db1", "k_dw2", "k_db2"):
        assert torch.equal(getattr(g1["dmlp"], n), getattr(g0["dmlp"], n)), f"{tag}: {n}"
    checks = [check_close(to_np(g1["dqkv"][..., 0, :, :]), to_np(g0["dqkv"][..., 0, :, :]),
                          f"{tag}: dQc"),
              check_close(to_np(g1["dqp"]), to_np(g0["dqp"]), f"{tag}: dQp", normalize=True)]
    for n in ("q_dw1", "q_db1", "q_dw2", "q_db2"):
        checks.append(check_close(to_np(getattr(g1["dmlp"], n)), to_np(getattr(g0["dmlp"], n)),
                                  f"{tag}: {n}", normalize=True))
    assert_all(checks)


@pytest.mark.parametrize("name", ["tiny", "w32"])
def test_training_step_replays_from_a_cuda_graph(name):
    w, qkv, step = _step_fn(name)
    ref = step()
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    # warm up on a side stream, as stream capture wants, then capture once
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        captured = step()
    graph.replay()
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    _compare(captured, ref, f"{name} replay")
    # new inputs in place: the replay follows them
    qkv.copy_(I.make_qkv(w.batch, w.height, w.width, w.heads, w.head_dim, seed=77).cuda())
    graph.replay()
    torch.cuda.synchronize()
    ref2 = step()
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    _compare(captured, ref2, f"{name} replay on new inputs")
    assert not torch.equal(ref2[0], ref[0])
