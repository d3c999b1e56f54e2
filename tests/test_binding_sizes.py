"""Host checks of the Python binding, on the CPU: buffers handed to the
library must hold the elements the call touches and live on the device of
its other tensors.  With CPU tensors of the right sizes every call gets past
these checks and stops at the first pointer (they must be CUDA tensors); a
wrong size or device stops it earlier with RIB_ERR_ARG."""
import pytest
import torch

import rib_inputs as I
import windowed_attention_implicit_b200 as R
from windowed_attention_implicit_b200 import _abi

B, H, W, HEADS, D, M, S, RANK, HID, F = 1, 32, 32, 2, 32, 16, 8, 16, 8, 4
bf, f32 = torch.bfloat16, torch.float32


def _mlp(device="cpu"):
    mq = I.make_mlp(F, HID, HEADS, RANK, 1, 0)
    mk = I.make_mlp(F, HID, HEADS, RANK, 1, 1)
    return R.PositionMLP.from_params(I.default_freqs(F), mq, mk, HEADS, RANK, device=device)


def _cla(C):
    p = I.make_cla(C, 1)
    return R.ClaGate.from_params(p.w_dw, p.b_dw, p.w_pw, p.b_pw, device="cpu")


def _bufs():
    """The buffers a training step hands the library (shapes as bench.py
    allocates them), at a small size."""
    pshape = (HEADS, M, M, RANK)
    return dict(
        qkv=torch.zeros((B, H, W, 3, HEADS, D), dtype=bf),
        dout=torch.zeros((B, H, W, HEADS, D), dtype=bf),
        out=torch.zeros((B, H, W, HEADS, D), dtype=bf),
        lse=torch.zeros((B, HEADS, H, W), dtype=f32),
        qp=torch.zeros(pshape, dtype=f32), kp=torch.zeros(pshape, dtype=f32),
        q16=torch.zeros(pshape, dtype=bf), k16=torch.zeros(pshape, dtype=bf),
        dqp=torch.zeros(pshape, dtype=f32), dkp=torch.zeros(pshape, dtype=f32))


def _passes(fn, *a, **kw):
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        fn(*a, **kw)


def _rejects(fn, what, *a, **kw):
    with pytest.raises(R.RibError, match=what) as e:
        fn(*a, **kw)
    assert e.value.code == _abi.RIB_ERR_ARG


def test_forward_buffers():
    b = _bufs()
    fwd = R.rib_window_attn_fwd
    _passes(fwd, b["qkv"], M, S, b["q16"], b["k16"], out=b["out"], lse=b["lse"])
    _passes(fwd, b["qkv"], M, S, b["q16"], b["k16"], out=b["out"], lse=b["lse"],
            region_mask=True)
    _passes(fwd, b["qkv"], M, S, None, None, rank=0)            # no position tokens
    _passes(fwd, b["qkv"], M, S, b["q16"][:, :, :, :0], None, rank=0)
    _rejects(fwd, "out holds", b["qkv"], M, S, b["q16"], b["k16"], out=b["out"][:, :16])
    _rejects(fwd, "lse holds", b["qkv"], M, S, b["q16"], b["k16"], lse=b["lse"][:, :1])
    # position tokens of another window size
    small = torch.zeros((HEADS, 8, 8, RANK), dtype=bf)
    _rejects(fwd, "qp_bf16 holds", b["qkv"], M, S, small, b["k16"])
    _rejects(fwd, "kp_bf16 holds", b["qkv"], M, S, b["q16"], small)
    _rejects(fwd, "qp_bf16 holds", b["qkv"], 32, 0, b["q16"], b["k16"])
    _rejects(fwd, "is on meta", b["qkv"], M, S, b["q16"], b["k16"],
             out=torch.empty(b["out"].shape, dtype=bf, device="meta"))


def test_forward_with_gate_buffers():
    b = _bufs()
    gate = torch.zeros((B, H, W, HEADS * D), dtype=bf)
    f = R.rib_window_attn_fwd_cla
    _passes(f, b["qkv"], M, S, gate, b["q16"], b["k16"], out=b["out"],
            out_gated=torch.empty_like(b["out"]), lse=b["lse"])
    _rejects(f, "out_gated holds", b["qkv"], M, S, gate, b["q16"], b["k16"],
             out_gated=b["out"][:, :8])
    _rejects(f, "qp_bf16 holds", b["qkv"], M, S, gate, b["q16"][:1], b["k16"])


def test_backward_buffers():
    b = _bufs()
    mlp = _mlp()
    dmlp = R.PositionMLPGrad.empty_like(mlp)
    bwd = R.rib_window_attn_bwd
    kw = dict(mlp=mlp, dqkv=torch.empty_like(b["qkv"]), dqp=b["dqp"], dkp=b["dkp"], dmlp=dmlp)
    _passes(bwd, b["qkv"], b["out"], b["dout"], b["lse"], M, S, b["q16"], b["k16"], **kw)
    _passes(bwd, b["qkv"], b["out"], b["dout"], b["lse"], M, S, b["q16"], b["k16"],
            region_mask=True, **kw)
    _passes(bwd, b["qkv"], b["out"], b["dout"], b["lse"], M, S, None, None, rank=0)
    _rejects(bwd, "dout holds", b["qkv"], b["out"], b["dout"][:, :1], b["lse"], M, S,
             b["q16"], b["k16"])
    _rejects(bwd, "dqkv holds", b["qkv"], b["out"], b["dout"], b["lse"], M, S, b["q16"],
             b["k16"], dqkv=b["out"])
    _rejects(bwd, "dkp holds", b["qkv"], b["out"], b["dout"], b["lse"], M, S, b["q16"],
             b["k16"], dkp=b["dkp"][:, :8])
    bad = R.PositionMLPGrad(*[t for t in dmlp.tensors().values()][:7], torch.empty(3))
    _rejects(bwd, "dmlp.k_db2 holds", b["qkv"], b["out"], b["dout"], b["lse"], M, S, b["q16"],
             b["k16"], mlp=mlp, dmlp=bad)


def test_position_token_buffers():
    b = _bufs()
    mlp = _mlp()
    _passes(R.rib_pos_tokens, mlp, M, b["qp"], b["kp"], b["q16"], b["k16"])
    _passes(R.rib_pos_tokens, mlp, M)
    _rejects(R.rib_pos_tokens, "kp holds", mlp, M, b["qp"], b["kp"][:1])
    _rejects(R.rib_pos_tokens, "qp_bf16 holds", mlp, 32, qp_bf16=b["q16"])
    dmlp = R.PositionMLPGrad.empty_like(mlp)
    _passes(R.rib_pos_tokens_bwd, mlp, M, b["dqp"], b["dkp"], dmlp)
    _passes(R.rib_pos_tokens_bwd_noalloc, mlp, M, b["dqp"], b["dkp"], dmlp)
    _rejects(R.rib_pos_tokens_bwd, "dqp holds", mlp, 32, b["dqp"], b["dkp"])
    bad = R.PositionMLPGrad(torch.empty(2), *list(dmlp.tensors().values())[1:])
    _rejects(R.rib_pos_tokens_bwd_noalloc, "dmlp.q_dw1 holds", mlp, M, b["dqp"], b["dkp"], bad)


def test_cla_buffers():
    C = HEADS * D
    cla = _cla(C)
    x = torch.zeros((B, H, W, C), dtype=bf)
    o = torch.zeros((B, H, W, HEADS, D), dtype=bf)
    _passes(R.rib_cla_gate, x, cla, gate=torch.empty_like(x))
    _rejects(R.rib_cla_gate, "gate holds", x, cla, gate=x[:, :8])
    _rejects(R.rib_cla_gate, "w_dw holds", x, _cla(96))
    gate = torch.empty_like(x)
    _passes(R.rib_cla_bwd, x, cla, gate, o, torch.empty_like(o), dout=torch.empty_like(o),
            dx=torch.empty_like(x))
    _rejects(R.rib_cla_bwd, "dout_gated holds", x, cla, gate, o, o[:, :4])
    _rejects(R.rib_cla_bwd, "dx holds", x, cla, gate, o, o, dx=x[:, :, :8])


def test_gather_scatter_buffers():
    C = 96
    x = torch.zeros((B, H, W, C), dtype=bf)
    nW = (H // M) * (W // M)
    xw = torch.zeros((B, nW, M * M, C), dtype=bf)
    _passes(R.rib_window_gather, x, M, S, out=xw)
    _passes(R.rib_window_scatter, xw, H, W, M, S, out=torch.empty_like(x))
    _rejects(R.rib_window_gather, "out holds", x, M, S, out=xw[:, :2])
    _rejects(R.rib_window_scatter, "out holds", xw, H, W, M, S, out=x[:, :16])
    # windows of another size than the call's
    _rejects(R.rib_window_scatter, "xw is", torch.zeros((B, 16, 64, C), dtype=bf), H, W, M, S)


def test_tensors_off_the_current_device_are_refused(monkeypatch):
    # the library launches on the current device; a call whose tensors live
    # on another GPU is refused before any pointer is handed over
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    with pytest.raises(R.RibError, match="current device is cuda:0") as e:
        R._sizes("rib_window_attn_fwd", torch.device("cuda", 1))
    assert e.value.code == _abi.RIB_ERR_ARG
    R._sizes("rib_window_attn_fwd", torch.device("cuda", 0))
    R._sizes("rib_window_attn_fwd", torch.device("cpu"))
