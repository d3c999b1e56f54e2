"""GPU parity of the optional shifted-window region mask (the *_masked entry
points) against the oracle's masked forward and backward."""
import numpy as np
import pytest
import torch

import oracle as O
import windowed_attention_implicit_b200 as R
from tests.rib_testlib import Case, assert_all, assert_close, check_close, to_np

pytestmark = pytest.mark.gpu

MASK_CASES = [
    # B, H, W, heads, M, s, rank
    (1, 64, 64, 2, 32, 16, 16),     # 4 windows, 3 of them hold several regions
    (2, 32, 48, 2, 16, 8, 16),      # H != W; the column band splits 16-wide key tiles
    (1, 64, 64, 1, 32, 8, 16),      # band boundary inside a 16-column tile (M - s = 24)
    (1, 96, 96, 1, 48, 40, 16),     # 3 x 3 windows, narrow wrapped band
    (1, 64, 64, 2, 32, 16, 0),      # rank 0
]


def _ids(c):
    return "B{}_H{}_W{}_h{}_M{}_s{}_r{}".format(*c)


@pytest.mark.parametrize("case", MASK_CASES, ids=[_ids(c) for c in MASK_CASES])
def test_masked_fwd_bwd_parity(case, bwd_kernel):
    B, H, W, heads, M, s, rank = case
    c = Case(B, H, W, heads, M, s, rank=rank, seed=21)
    d = c.device()
    out, lse = R.rib_window_attn_fwd(d["qkv"], M, s, d["qp16"], d["kp16"], rank=rank,
                                     region_mask=True)
    g = R.rib_window_attn_bwd(d["qkv"], out, d["dout"], lse, M, s, d["qp16"], d["kp16"],
                              rank=rank, region_mask=True)
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    ro, rl = O.attn_fwd(c.qkv, M, s, c.qp16, c.kp16, c.scale, region_mask=True)
    dq, dqp, dkp = O.attn_bwd(c.qkv, c.dout, M, s, c.qp16, c.kp16, c.scale, region_mask=True)
    # the mask really changes these cases
    uo, _ = O.attn_fwd(c.qkv, M, s, c.qp16, c.kp16, c.scale)
    assert np.abs(uo - ro).max() > 0.05
    got = to_np(g["dqkv"])
    checks = [check_close(to_np(out), ro, "out"), check_close(to_np(lse), rl, "lse")]
    checks += [check_close(got[:, :, :, k], dq[:, :, :, k], name)
               for k, name in enumerate(("dQc", "dKc", "dV"))]
    if rank:
        checks += [check_close(to_np(g["dqp"]), dqp, "dQp", normalize=True),
                   check_close(to_np(g["dkp"]), dkp, "dKp", normalize=True)]
    assert_all(checks)


def test_mask_changes_only_multi_region_windows_and_nothing_without_shift():
    """Interior windows take the unmasked code path: bit-identical output.
    With shift 0 the mask is empty: identical to the unmasked call."""
    c = Case(1, 64, 96, 2, 32, 16, seed=5)
    d = c.device()
    o0, l0 = R.rib_window_attn_fwd(d["qkv"], 32, 16, d["qp16"], d["kp16"])
    o1, l1 = R.rib_window_attn_fwd(d["qkv"], 32, 16, d["qp16"], d["kp16"], region_mask=True)
    torch.cuda.synchronize()
    H, W, M, s = 64, 96, 32, 16
    ry = (np.arange(H) - s) % H
    rx = (np.arange(W) - s) % W
    interior = torch.tensor((ry[:, None] < H - M) & (rx[None, :] < W - M))
    assert torch.equal(o0[0][interior], o1[0][interior])
    assert not torch.equal(o0[0][~interior], o1[0][~interior])
    c0 = Case(1, 64, 64, 2, 32, 0, seed=6)
    d0 = c0.device()
    a, la = R.rib_window_attn_fwd(d0["qkv"], 32, 0, d0["qp16"], d0["kp16"])
    b, lb = R.rib_window_attn_fwd(d0["qkv"], 32, 0, d0["qp16"], d0["kp16"], region_mask=True)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_masked_full_size_sampled_rows():
    """The 96 x 96-window workload (192 x 192 map, shift 48): sampled query rows
    of every window of one head against the oracle's masked rows."""
    c = Case(1, 192, 192, 1, 96, 48, seed=9)
    d = c.device()
    out, lse = R.rib_window_attn_fwd(d["qkv"], 96, 48, d["qp16"], d["kp16"], region_mask=True)
    torch.cuda.synchronize()
    assert R.rib_last_status()[0] == 0
    out, lse = to_np(out), to_np(lse)
    rng = np.random.default_rng(3)
    checks = []
    for w in range(4):
        wy, wx = divmod(w, 2)
        lab = O.region_labels(192, 192, 96, 48, wy, wx)
        rows = np.sort(rng.choice(96 * 96, 96, replace=False))
        qc, kc, v, qpf, kpf = O.gather_unit(c.qkv, c.qp16, c.kp16, 96, 48, 0, w, 0)
        ro, rl = O.attention_unit_rows(qc, kc, v, qpf, kpf, c.scale, rows=rows, labels=lab)
        y = (wy * 96 + rows // 96 + 48) % 192
        x = (wx * 96 + rows % 96 + 48) % 192
        checks.append(check_close(out[0, y, x, 0], ro, f"out window {w}"))
        checks.append(check_close(lse[0, 0, y, x], rl, f"lse window {w}"))
    assert_all(checks)
