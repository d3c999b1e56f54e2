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
