"""The data-parallel path on CPU: 2 gloo ranks each take a batch shard, compute
their partial position-MLP gradients (with the oracle, standing in for the
CUDA kernels) and sum them with the package's all-reduce; the result must
equal the single-process gradient over the whole batch."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
import rib_inputs as I
from windowed_attention_implicit_b200.parallel import FlatGrads, allreduce_grads, shard_batch

B, H, W, HEADS, M, S, R, HID, F = 3, 16, 16, 2, 8, 4, 4, 6, 3


def _inputs():
    qkv = I.make_qkv(B, H, W, HEADS, 5, seed=21)
    dout = I.make_dout(B, H, W, HEADS, 5, seed=21)
    freqs = I.default_freqs(F)
    mq = I.make_mlp(F, HID, HEADS, R, 21, 0, strong=True)
    mk = I.make_mlp(F, HID, HEADS, R, 21, 1, strong=True)
    return qkv, dout, freqs, mq, mk


def _grads(qkv, dout, freqs, mq, mk):
    qp, kp = O.pos_tokens(freqs, mq, mk, M, HEADS, R)
    _, dqp, dkp = O.attn_bwd(qkv, dout, M, S, qp, kp)
    gq, gk = O.pos_tokens_backward(freqs, mq, mk, M, dqp, dkp)
    return list(gq) + list(gk)


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        qkv, dout, freqs, mq, mk = _inputs()
        sl = shard_batch(B, world, rank)
        local = _grads(qkv[sl], dout[sl], freqs, mq, mk)
        fg = FlatGrads([g.shape for g in local], device="cpu", dtype=torch.float64)
        for v, g in zip(fg.views, local):
            v.copy_(torch.from_numpy(g))
        allreduce_grads(fg.flat)
        if rank == 0:
            q.put([v.numpy().copy() for v in fg.views])
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_shard_batch_covers_everything_once():
    for gb in range(0, 9):
        for world in range(1, 5):
            seen = []
            for r in range(world):
                sl = shard_batch(gb, world, r)
                seen.extend(range(gb)[sl])
            assert seen == list(range(gb))


def test_two_rank_gloo_allreduce_matches_single_process():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = q.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ref = _grads(*_inputs())
    for g, r in zip(got, ref):
        assert np.allclose(g, r, rtol=1e-12, atol=1e-12)


# With the convolutional local attention gate in the step, its weight
# gradients (sums over every pixel) share the MLP gradients' buffer: still one
# all-reduce per step.
C_CLA = HEADS * 5


def _cla_inputs():
    x = I.make_features(B, H, W, C_CLA, seed=31).float().numpy()
    o = I.make_features(B, H, W, C_CLA, seed=32).float().numpy()
    dog = I.make_features(B, H, W, C_CLA, seed=33).float().numpy()
    return x, o, dog, I.make_cla(C_CLA, seed=31)


def _cla_grads(x, o, dog, p):
    from oracle.cla_oracle import cla_backward
    g = cla_backward(x, p.w_dw.numpy(), p.b_dw.numpy(), p.w_pw.numpy(), p.b_pw.numpy(), o, dog)
    return [g["dw_dw"], g["db_dw"], g["dw_pw"], g["db_pw"]]


def _worker_mlp_cla(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        qkv, dout, freqs, mq, mk = _inputs()
        x, o, dog, p = _cla_inputs()
        sl = shard_batch(B, world, rank)
        local = _grads(qkv[sl], dout[sl], freqs, mq, mk) + _cla_grads(x[sl], o[sl], dog[sl], p)
        fg = FlatGrads([g.shape for g in local], device="cpu", dtype=torch.float64,
                       names=FlatGrads.ORDER + FlatGrads.CLA_ORDER)
        for v, g in zip(fg.views, local):
            v.copy_(torch.from_numpy(np.ascontiguousarray(g)))
        allreduce_grads(fg.flat)
        if rank == 0:
            q.put([v.numpy().copy() for v in fg.views])
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_allreduce_with_cla_gradients():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_mlp_cla, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = q.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ref = _grads(*_inputs()) + _cla_grads(*_cla_inputs())
    assert len(got) == len(ref) == 12
    for g, r in zip(got, ref):
        assert g.shape == r.shape
        assert np.allclose(g, r, rtol=1e-12, atol=1e-12)
    # a shard's CLA gradient alone is not the whole sum
    part = _cla_grads(*(a[:1] for a in _cla_inputs()[:3]), _cla_inputs()[3])
    assert not np.allclose(part[2], ref[10])


def test_flat_layouts():
    from windowed_attention_implicit_b200 import PositionMLP
    mq = I.make_mlp(F, HID, HEADS, R, 21, 0)
    mk = I.make_mlp(F, HID, HEADS, R, 21, 1)
    mlp = PositionMLP(torch.tensor([1.0]),
                      *(t.contiguous() for t in (mq.w1, mq.b1, mq.w2, mq.b2,
                                                 mk.w1, mk.b1, mk.w2, mk.b2)), HEADS, R)
    both = FlatGrads.for_mlp_and_cla(mlp, C_CLA)
    n_mlp = sum(t.numel() for t in (mq.w1, mq.b1, mq.w2, mq.b2, mk.w1, mk.b1, mk.w2, mk.b2))
    assert both.flat.numel() == n_mlp + 9 * C_CLA + C_CLA + C_CLA * C_CLA + C_CLA
    assert tuple(both.cla()["dw_dw"].shape) == (C_CLA, 3, 3)
    assert tuple(both.cla()["dw_pw"].shape) == (C_CLA, C_CLA)
    assert both.as_grad().q_dw1.shape == mq.w1.shape
    both.cla()["db_pw"].fill_(2.0)                  # views of the one buffer
    assert both.flat[-C_CLA:].eq(2.0).all()
    with pytest.raises(ValueError):
        FlatGrads.for_cla(C_CLA, "cpu").as_grad()
    with pytest.raises(ValueError):
        FlatGrads.for_mlp(mlp).cla()
    with pytest.raises(ValueError):
        FlatGrads([(2,), (3,)], "cpu", names=("a",))
