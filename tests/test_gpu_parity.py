"""GPU parity: every CUDA entry point against the fp64 oracle (small sizes
that span several tiles, odd tile counts and the shift / rank edge cases)."""
import numpy as np
import pytest
import torch

import oracle as O
import rib_inputs as I
import windowed_attention_implicit_b200 as R
from tests.rib_testlib import (Case, assert_all, assert_close, bf16_round, check_close,
                               mlp_grad_checks, stats, to_np, POS_REL)

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------- pos tokens

@pytest.mark.parametrize("M", [1, 5, 16, 32, 96])
@pytest.mark.parametrize("strong", [False, True])
def test_pos_tokens_parity(M, strong):
    heads, rank, hid, F = 6, 16, 128, 16
    freqs = I.default_freqs(F)
    mq = I.make_mlp(F, hid, heads, rank, 7, 0, strong=strong)
    mk = I.make_mlp(F, hid, heads, rank, 7, 1, strong=strong)
    mlp = R.PositionMLP.from_params(freqs, mq, mk, heads, rank)
    qp, kp, q16, k16 = R.rib_pos_tokens(mlp, M)
    torch.cuda.synchronize()
    rq, rk = O.pos_tokens(freqs, mq, mk, M, heads, rank)
    for got, ref, name in ((qp, rq, "qp"), (kp, rk, "kp")):
        g = to_np(got)
        rel = np.abs(g - ref).max() / np.abs(ref).max()
        assert rel <= POS_REL, f"{name} M={M}: rel {rel:.3e}"
    # bf16 copies are the round-to-nearest-even of the fp32 result
    assert torch.equal(q16.cpu(), qp.cpu().to(torch.bfloat16))
    assert torch.equal(k16.cpu(), kp.cpu().to(torch.bfloat16))


# Shapes for both kernel forms: the register-tiled one (hid % 8 == 0,
# rank % 8 == 0) and the general one (the other shapes).
MLP_SHAPES = [  # heads, rank, hid, F
    (4, 12, 60, 16),    # general: hid and rank not multiples of 8
    (3, 6, 36, 8),      # general
    (2, 8, 64, 5),      # tiled, 20 Fourier inputs
    (1, 16, 8, 1),      # tiled, smallest
]


@pytest.mark.parametrize("heads,rank,hid,F", MLP_SHAPES)
def test_pos_tokens_parity_both_kernel_forms(heads, rank, hid, F):
    M = 12
    freqs = I.default_freqs(F)
    mq = I.make_mlp(F, hid, heads, rank, 31, 0, strong=True)
    mk = I.make_mlp(F, hid, heads, rank, 31, 1, strong=True)
    mlp = R.PositionMLP.from_params(freqs, mq, mk, heads, rank)
    qp, kp, q16, k16 = R.rib_pos_tokens(mlp, M)
    torch.cuda.synchronize()
    rq, rk = O.pos_tokens(freqs, mq, mk, M, heads, rank)
    for got, ref, name in ((qp, rq, "qp"), (kp, rk, "kp")):
        rel = np.abs(to_np(got) - ref).max() / np.abs(ref).max()
        assert rel <= POS_REL, f"{name}: rel {rel:.3e}"
    assert torch.equal(q16.cpu(), qp.cpu().to(torch.bfloat16))


# ---------------------------------------------------------------- gather/scatter

@pytest.mark.parametrize("B,H,W,C,dtype,M,s", [
    (1, 16, 16, 8, torch.int16, 8, 0),
    (2, 32, 48, 96, torch.bfloat16, 16, 8),
    (1, 64, 64, 576, torch.bfloat16, 32, 16),
    (3, 24, 40, 4, torch.float32, 8, 0),
    (1, 96, 96, 16, torch.uint8, 48, 40),
    (1, 192, 192, 192, torch.bfloat16, 96, 48),
])
def test_window_gather_scatter_bit_exact(B, H, W, C, dtype, M, s):
    g = torch.Generator().manual_seed(B * 1000 + C)
    raw = torch.randint(0, 255, (B, H, W, C * torch.tensor([], dtype=dtype).element_size()),
                        dtype=torch.uint8, generator=g)
    x = raw.view(dtype).reshape(B, H, W, C)
    xd = x.cuda()
    xw = R.rib_window_gather(xd, M, s)
    back = R.rib_window_scatter(xw, H, W, M, s)
    torch.cuda.synchronize()
    ref = O.window_partition(x.view(torch.uint8).numpy(), M, s)   # byte view: exact
    got = xw.cpu().view(torch.uint8).numpy()
    assert np.array_equal(got, ref.reshape(got.shape))
    assert torch.equal(back.cpu().view(torch.uint8), x.view(torch.uint8))


# ---------------------------------------------------------------- attention

FWD_CASES = [
    # B, H, W, heads, M, s, rank, strong
    (1, 64, 64, 3, 16, 0, 16, False),     # the tiny workload
    (1, 64, 64, 3, 16, 0, 16, True),      # strong positional bias
    (1, 64, 64, 2, 32, 16, 16, True),     # shifted, 8 tiles per unit
    (2, 32, 48, 2, 16, 8, 16, True),      # H != W, shift of half a box
    (1, 96, 96, 1, 48, 24, 16, True),     # 3 tiles per tile row, 18 tiles
    (1, 64, 64, 2, 32, 0, 0, True),       # rank 0: plain windowed attention
    (1, 128, 128, 1, 64, 56, 16, True),   # largest shift < M
    (1, 96, 96, 2, 96, 0, 16, True),      # 96x96 window, no shift
    (1, 96, 192, 1, 96, 72, 16, True),    # H != W, shift 72: boxes wrap at the map edge
    (1, 96, 96, 1, 48, 0, 0, True),       # rank 0, 18 tiles per unit
    (1, 96, 96, 1, 48, 8, 16, True),      # shift of one box
]


def _ids(c):
    return "B{}H{}W{}h{}M{}s{}r{}{}".format(*c[:7], "S" if c[7] else "")


@pytest.mark.parametrize("case", FWD_CASES, ids=[_ids(c) for c in FWD_CASES])
def test_fwd_parity(case):
    B, H, W, heads, M, s, rank, strong = case
    c = Case(B, H, W, heads, M, s, rank=rank, strong=strong, seed=11)
    d = c.device()
    out, lse = R.rib_window_attn_fwd(d["qkv"], M, s, d["qp16"], d["kp16"], rank=rank)
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    ro, rl = c.oracle_fwd()
    assert_close(to_np(out), ro, "out")
    assert_close(to_np(lse), rl, "lse")


def test_fwd_explicit_scale_and_default_agree():
    c = Case(1, 64, 64, 2, 32, 16, seed=5)
    d = c.device()
    o1, l1 = R.rib_window_attn_fwd(d["qkv"], 32, 16, d["qp16"], d["kp16"], scale=0.0)
    o2, l2 = R.rib_window_attn_fwd(d["qkv"], 32, 16, d["qp16"], d["kp16"], scale=c.scale)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    o3, l3 = R.rib_window_attn_fwd(d["qkv"], 32, 16, d["qp16"], d["kp16"], scale=0.3)
    ro, rl = O.attn_fwd(c.qkv, 32, 16, c.qp16, c.kp16, 0.3)
    assert_close(to_np(o3), ro, "out scale=0.3")
    assert_close(to_np(l3), rl, "lse scale=0.3")


@pytest.mark.parametrize("case", FWD_CASES, ids=[_ids(c) for c in FWD_CASES])
def test_bwd_parity(case, bwd_kernel):
    B, H, W, heads, M, s, rank, strong = case
    c = Case(B, H, W, heads, M, s, rank=rank, strong=strong, seed=13)
    d = c.device()
    out, lse = R.rib_window_attn_fwd(d["qkv"], M, s, d["qp16"], d["kp16"], rank=rank)
    g = R.rib_window_attn_bwd(d["qkv"], out, d["dout"], lse, M, s, d["qp16"], d["kp16"],
                              rank=rank)
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    dq, dqp, dkp = c.oracle_bwd()
    got = to_np(g["dqkv"])
    checks = [check_close(got[:, :, :, k], dq[:, :, :, k], name)
              for k, name in enumerate(("dQc", "dKc", "dV"))]
    if rank:
        checks.append(check_close(to_np(g["dqp"]), dqp, "dQp", normalize=True))
        checks.append(check_close(to_np(g["dkp"]), dkp, "dKp", normalize=True))
    assert_all(checks)


def test_bwd_mlp_grads_parity(bwd_kernel):
    """Training step of the w32 shape at reduced batch: MLP weight grads from
    the kernel chain (pos tokens -> attention bwd -> MLP bwd) vs the oracle."""
    B, H, W, heads, M, s = 1, 64, 64, 6, 32, 16
    c = Case(B, H, W, heads, M, s, hidden=128, seed=17, strong=True)
    mlp = R.PositionMLP.from_params(c.freqs, c.mlp_q, c.mlp_k, heads, 16)
    d = c.device()
    out, lse = R.rib_window_attn_fwd(d["qkv"], M, s, d["qp16"], d["kp16"])
    g = R.rib_window_attn_bwd(d["qkv"], out, d["dout"], lse, M, s, d["qp16"], d["kp16"],
                              mlp=mlp)
    torch.cuda.synchronize()
    _, dqp, dkp = c.oracle_bwd()
    (gq, gk) = O.pos_tokens_backward(c.freqs, c.mlp_q, c.mlp_k, M, dqp, dkp)
    dm = g["dmlp"]
    checks = [check_close(to_np(g["dqp"]), dqp, "dQp", normalize=True), check_close(to_np(g["dkp"]), dkp, "dKp", normalize=True)]
    checks += mlp_grad_checks(dm, gq, gk)
    assert_all(checks)


MLP_REL = 1e-4   # fp32 sums over up to 9216 tokens: ~sqrt(n) * 6e-8 relative, with margin


@pytest.mark.parametrize("M,hid", [(16, 64), (32, 128), (96, 128), (5, 32)])
def test_pos_tokens_bwd_parity(M, hid):
    """The position-MLP backward alone, from seeded dL/dQp, dL/dKp."""
    heads, rank, F = 6, 16, 16
    freqs = I.default_freqs(F)
    mq = I.make_mlp(F, hid, heads, rank, 23, 0, strong=True)
    mk = I.make_mlp(F, hid, heads, rank, 23, 1, strong=True)
    mlp = R.PositionMLP.from_params(freqs, mq, mk, heads, rank)
    gq = I.randn((heads, M, M, rank), seed=M, tag=7)
    gk = I.randn((heads, M, M, rank), seed=M, tag=8)
    dm = R.rib_pos_tokens_bwd(mlp, M, gq.cuda(), gk.cuda())
    torch.cuda.synchronize()
    (rq, rk) = O.pos_tokens_backward(freqs, mq, mk, M, gq.double().numpy(), gk.double().numpy())
    bad = []
    for side, ref in (("q", rq), ("k", rk)):
        for name, r in zip(("dw1", "db1", "dw2", "db2"), ref):
            got = to_np(getattr(dm, f"{side}_{name}"))
            rel = np.abs(got - r).max() / np.abs(r).max()
            print(f"{side}_{name}: rel {rel:.3e}")
            if rel > MLP_REL:
                bad.append(f"{side}_{name} rel {rel:.3e}")
    assert not bad, bad


@pytest.mark.parametrize("heads,rank,hid,F", MLP_SHAPES)
def test_pos_tokens_bwd_parity_both_kernel_forms(heads, rank, hid, F):
    M = 20   # 400 tokens: seven chunks of 64, the last one partial
    freqs = I.default_freqs(F)
    mq = I.make_mlp(F, hid, heads, rank, 37, 0, strong=True)
    mk = I.make_mlp(F, hid, heads, rank, 37, 1, strong=True)
    mlp = R.PositionMLP.from_params(freqs, mq, mk, heads, rank)
    gq = I.randn((heads, M, M, rank), seed=M, tag=7)
    gk = I.randn((heads, M, M, rank), seed=M, tag=8)
    dm = R.rib_pos_tokens_bwd(mlp, M, gq.cuda(), gk.cuda())
    torch.cuda.synchronize()
    (rq, rk) = O.pos_tokens_backward(freqs, mq, mk, M, gq.double().numpy(), gk.double().numpy())
    bad = []
    for side, ref in (("q", rq), ("k", rk)):
        for name, r in zip(("dw1", "db1", "dw2", "db2"), ref):
            rel = np.abs(to_np(getattr(dm, f"{side}_{name}")) - r).max() / np.abs(r).max()
            if rel > MLP_REL:
                bad.append(f"{side}_{name} rel {rel:.3e}")
    assert not bad, bad


# ---------------------------------------------------------------- status

def test_bounded_wait_records_timeout_and_context_survives():
    R.rib_last_status()                           # clear
    R.rib_debug_wait_timeout(2_000_000)           # 2 ms, nothing arrives
    code, site = R.rib_last_status()
    assert code == R._abi.RIB_ERR_TIMEOUT and site == 1
    assert R.rib_last_status()[0] == 0            # cleared by the read
    c = Case(1, 32, 32, 1, 16, 0, seed=3)         # the context is still usable
    d = c.device()
    out, lse = R.rib_window_attn_fwd(d["qkv"], 16, 0, d["qp16"], d["kp16"])
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    ro, _ = c.oracle_fwd()
    assert_close(to_np(out), ro, "out after timeout")


def test_fma_pipe_exp2_error_bound():
    """The forward kernel's FMA-pipe exp2 against fp64 2^x: relative error
    within the polynomial's minimax bound (7.48e-5, fit_exp2_poly.py) plus
    fp32 rounding, over the range the softmax feeds it ([-125, 8]); below
    -125 the input is clamped, giving at most 2^-125."""
    g = torch.Generator().manual_seed(3)
    x = torch.cat([torch.linspace(-125.0, 8.0, 200_000),
                   torch.rand(100_000, generator=g) * -20.0,
                   torch.tensor([0.0, -0.5, 0.5, -1.0, 1.0, 7.999, -124.5, -300.0])])
    if x.numel() % 2:
        x = torch.cat([x, torch.tensor([0.25])])
    y = R.rib_debug_exp2(x.cuda()).cpu().double()
    xd = x.double()
    ref = torch.exp2(xd)
    ok = xd >= -125.0
    rel = ((y[ok] - ref[ok]).abs() / ref[ok]).max().item()
    print(f"max relative error {rel:.3e}")
    assert rel <= 7.6e-5
    assert (y[~ok] <= 2.0 ** -124).all() and (y[~ok] >= 0).all()
