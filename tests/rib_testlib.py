"""Shared helpers of the parity tests: inputs, oracle runs, comparisons.

Inputs come from rib_inputs (seeded); expected values only from oracle/.
The attention parity cases feed both sides the same bf16-rounded Qp/Kp (the
oracle computes them in fp64, the host rounds them), so each kernel is
compared on exactly the values it consumes.
"""
from __future__ import annotations

import re

import numpy as np
import torch

import oracle as O
import rib_inputs as I

MAX_ABS = 2e-2     # outputs and gradients, bf16 in / fp32 accumulate
MEAN_ABS = 2e-3
POS_REL = 1e-5     # Qp/Kp fp32: max|d| / max|ref|


def tf32_error_bounds(qkv, qp, kp, M, s, tau, row_block=512):
    """First-order elementwise error bounds of the fp32 forward on the tf32
    tensor cores against the exact result, from tf32's 10 explicit mantissa
    bits.  Per unit, with augmented rows q_i = [Qc_i, Qp_i], k_j = [Kc_j, Kp_j]:

      the MMA reads every operand as tf32: |relative error| <= 2^-10 each
      (2^-10 whether it truncates or rounds), so a logit s_ij = tau q_i.k_j
      is off by at most  e_ij = (2 * 2^-10 + 48 * 2^-24) tau sum_k |q_ik k_jk|
      (the second term: fp32 accumulation of 48 products);
      lse_i = ln sum_j exp(s_ij) moves by at most max_j e_ij;
      P is perturbed by e_ij, by its rounding to tf32 (2^-11, to nearest) and
      by the hardware exp2 (< 2^-20); V by 2^-10; to first order
        |dO_ic| <= sum_j P_ij (e_ij + 2^-11 + 2^-20) |v_jc - O_ic|
                   + (2^-10 + N 2^-24) sum_j P_ij |v_jc|.

    Returns (out_bound [B][H][W][heads][d], lse_bound [B][heads][H][W]) at
    the map's pixels, computed in fp64 from the same inputs as the oracle."""
    x = O.window_partition(np.asarray(qkv, dtype=np.float64), M, s)
    B, nW, N, _, heads, d = x.shape
    qp = np.asarray(qp, dtype=np.float64).reshape(heads, N, -1)
    kp = np.asarray(kp, dtype=np.float64).reshape(heads, N, -1)
    r = qp.shape[-1]
    ob = np.empty((B, nW, N, heads, d))
    lb = np.empty((B, nW, N, heads))
    e_log = 2.0 ** -9 + (d + r) * 2.0 ** -24
    for b in range(B):
        for w in range(nW):
            for h in range(heads):
                qa = np.concatenate([x[b, w, :, 0, h], qp[h]], 1)
                ka = np.concatenate([x[b, w, :, 1, h], kp[h]], 1)
                v = x[b, w, :, 2, h]
                for r0 in range(0, N, row_block):
                    r1 = min(N, r0 + row_block)
                    e = e_log * tau * (np.abs(qa[r0:r1]) @ np.abs(ka).T)
                    sc = tau * (qa[r0:r1] @ ka.T)
                    pm = np.exp(sc - sc.max(1, keepdims=True))
                    pm /= pm.sum(1, keepdims=True)
                    o = pm @ v
                    lb[b, w, r0:r1, h] = e.max(1)
                    ep = pm * (e + 2.0 ** -11 + 2.0 ** -20)
                    dev = np.abs(v[None, :, :] - o[:, None, :])       # [rows, N, d]
                    ob[b, w, r0:r1, h] = (np.einsum("ij,ijc->ic", ep, dev) +
                                          (2.0 ** -10 + N * 2.0 ** -24) * (pm @ np.abs(v)))
    H, W = np.asarray(qkv).shape[1:3]
    out_b = O.window_reverse(ob, M, s, H, W)
    lse_b = O.window_reverse(lb, M, s, H, W).transpose(0, 3, 1, 2)
    # second-order terms and the few ulps of the fp32 rescales: 5 % + 1e-6
    return 1.05 * out_b + 1e-6, 1.05 * lse_b + 1e-6


def check_within_bound(got, ref, bound, what):
    """'' if |got - ref| <= bound elementwise, else a message; prints the
    largest ratio of error to bound."""
    err = np.abs(np.asarray(got, dtype=np.float64) - np.asarray(ref, dtype=np.float64))
    ratio = float((err / bound).max()) if err.size else 0.0
    msg = f"{what}: max |d| / bound = {ratio:.3f} (max |d| {err.max():.3e}, max bound {bound.max():.3e})"
    print(msg)
    RECORDS.append({"what": what + " (tf32 bound)", "max_abs": float(err.max()),
                    "mean_abs": float(err.mean()), "max_ref": float(np.abs(ref).max()),
                    "abs_within": ratio <= 1.0, "normalised_by": None, "within": ratio <= 1.0})
    return "" if ratio <= 1.0 else msg


def stats(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = np.abs(got - ref)
    return float(d.max()) if d.size else 0.0, float(d.mean()) if d.size else 0.0


# Tensors whose error may be judged relative to their magnitude (besides the
# absolute figure, which is always computed and reported): fp32 sums over
# windows or tokens (dQp, dKp, the position-MLP and CLA weight gradients) and
# the CLA's dO = dO' * G, which carries the upstream gradient's magnitude.
NORMALISED = {"dqp", "dkp", "dw1", "db1", "dw2", "db2", "dw", "db", "do"}

# every comparison made in this process: name, absolute and normalised
# figures (written out as JSON lines when RIB_PARITY_LOG names a file)
RECORDS = []


def check_close(got, ref, what, max_abs=MAX_ABS, mean_abs=MEAN_ABS, normalize=False,
                grown_inputs=False):
    """Returns an error message ('' if within bounds).

    The absolute max/mean errors are always computed, reported and recorded.
    normalize=True divides the errors by max(1, max|ref|) before the bounds
    are applied, and a number divides them by max(1, that number).  It is
    allowed only for the tensors named in NORMALISED, whose magnitude grows
    with the number of windows or tokens summed, and for cases whose inputs
    are scaled up on purpose (grown_inputs=True)."""
    mx, mn = stats(got, ref)
    refmax = float(np.abs(np.asarray(ref, dtype=np.float64)).max()) if np.size(ref) else 0.0
    if normalize:
        tokens = set(re.split(r"[ _]", what.lower()))
        assert grown_inputs or tokens & NORMALISED, \
            f"{what}: a magnitude-relative bound is not allowed for this tensor"
    if normalize is True:
        scale = max(1.0, refmax)
    elif normalize:
        scale = max(1.0, float(normalize))
    else:
        scale = 1.0
    abs_ok = mx <= max_abs and mn <= mean_abs
    ok = mx / scale <= max_abs and mn / scale <= mean_abs
    msg = (f"{what}: abs max|d|={mx:.3e} mean|d|={mn:.3e} "
           f"({'within' if abs_ok else 'beyond'} {max_abs}/{mean_abs}), max|ref|={refmax:.3e}")
    if normalize:
        msg += (f"; normalised by {scale:.3e}: max {mx / scale:.3e} mean {mn / scale:.3e} "
                f"({'within' if ok else 'beyond'} bounds)")
    print(msg)
    RECORDS.append({"what": what, "max_abs": mx, "mean_abs": mn, "max_ref": refmax,
                    "abs_within": abs_ok, "normalised_by": scale if normalize else None,
                    "within": ok})
    return "" if ok else msg


def assert_close(got, ref, what, max_abs=MAX_ABS, mean_abs=MEAN_ABS, normalize=False):
    msg = check_close(got, ref, what, max_abs, mean_abs, normalize)
    assert not msg, msg


def assert_all(checks):
    """checks: list of messages from check_close; fails listing every miss."""
    bad = [c for c in checks if c]
    assert not bad, "; ".join(bad)


def mlp_grad_checks(dmlp, ref_q, ref_k):
    """Position-MLP weight grads of one side are measured against that side's common
    scale, max(1, max|ref| over its four tensors): the key MLP's output-bias
    gradient is a sum that cancels exactly (rows of dS sum to zero), so its
    own magnitude says nothing about the size of the terms summed."""
    checks = []
    for side, ref in (("q", ref_q), ("k", ref_k)):
        scale = max(float(np.abs(r).max()) for r in ref)
        for name, r in zip(("dw1", "db1", "dw2", "db2"), ref):
            checks.append(check_close(to_np(getattr(dmlp, f"{side}_{name}")), r,
                                      f"{side}_{name}", normalize=scale))
    return checks


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_round(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a), dtype=torch.float64).to(torch.bfloat16)


class Case:
    """One attention problem: host inputs, their device copies and the
    oracle's position tokens."""

    def __init__(self, B, H, W, heads, M, s, rank=16, hidden=64, F=16, seed=0,
                 strong=True, qkv_std=1.0):
        self.B, self.H, self.W, self.heads, self.M, self.s, self.rank = B, H, W, heads, M, s, rank
        self.d = 32
        self.qkv = I.make_qkv(B, H, W, heads, 32, seed, std=qkv_std)
        self.dout = I.make_dout(B, H, W, heads, 32, seed)
        self.freqs = I.default_freqs(F)
        r = max(rank, 1)
        self.mlp_q = I.make_mlp(F, hidden, heads, r, seed, 0, strong=strong)
        self.mlp_k = I.make_mlp(F, hidden, heads, r, seed, 1, strong=strong)
        if rank > 0:
            qp, kp = O.pos_tokens(self.freqs, self.mlp_q, self.mlp_k, M, heads, rank)
            self.qp16, self.kp16 = bf16_round(qp), bf16_round(kp)
        else:
            self.qp16 = torch.zeros((heads, M, M, 0), dtype=torch.bfloat16)
            self.kp16 = torch.zeros((heads, M, M, 0), dtype=torch.bfloat16)
        self.scale = O.default_scale(32, rank)

    def device(self):
        dev = "cuda"
        return dict(qkv=self.qkv.to(dev), dout=self.dout.to(dev),
                    qp16=self.qp16.to(dev) if self.rank else None,
                    kp16=self.kp16.to(dev) if self.rank else None)

    def oracle_fwd(self):
        return O.attn_fwd(self.qkv, self.M, self.s, self.qp16, self.kp16, self.scale)

    def oracle_bwd(self, units=None):
        return O.attn_bwd(self.qkv, self.dout, self.M, self.s, self.qp16, self.kp16,
                          self.scale, units=units)
