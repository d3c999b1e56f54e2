"""Runs every work entry point of the library once on seeded inputs and saves
the outputs, for the comparison of the release and debug builds
(tests/test_gpu_debug_build.py runs it twice, with and without
RIB_DEBUG_LIBRARY=1).

    python -m tests.debug_build_run OUT.npz

After each call the status word must be RIB_OK (in the debug build: no
guarded access fell outside its buffer).  Outputs whose sums run in a fixed
order are saved under their name; the query-side gradients of the attention
backward (fp32 sums in CTA-scheduling order) are saved with a "~" prefix.
"""
from __future__ import annotations

import ctypes
import sys

import numpy as np
import torch

import rib_inputs as I
import windowed_attention_implicit_b200 as R
from windowed_attention_implicit_b200 import _abi


def _np(t):
    return t.detach().float().cpu().numpy()


def main(path: str) -> None:
    out = {}
    calls = []

    def done(name):
        torch.cuda.synchronize()
        code, site = R.rib_last_status()
        calls.append(name)
        if code != 0:
            info = (ctypes.c_ulonglong * 2)()
            R.library().rib_debug_guard_info(info)
            raise SystemExit(f"{name}: status {R.rib_status_string(code)} at site {site}, "
                             f"index {info[0]} of {info[1]}")

    # position tokens and the MLP backward: register-tiled and general shapes
    for tag, (heads, rank, hid, F, M) in {"tiled": (6, 16, 128, 16, 32),
                                          "general": (4, 12, 60, 16, 20)}.items():
        mq = I.make_mlp(F, hid, heads, rank, 3, 0, strong=True)
        mk = I.make_mlp(F, hid, heads, rank, 3, 1, strong=True)
        mlp = R.PositionMLP.from_params(I.default_freqs(F), mq, mk, heads, rank)
        qp, kp, q16, k16 = R.rib_pos_tokens(mlp, M)
        done(f"rib_pos_tokens {tag}")
        out[f"qp_{tag}"], out[f"kp16_{tag}"] = _np(qp), _np(k16)
        gq = I.randn((heads, M, M, rank), seed=5, tag=7).cuda()
        gk = I.randn((heads, M, M, rank), seed=5, tag=8).cuda()
        dm = R.rib_pos_tokens_bwd(mlp, M, gq, gk)
        done(f"rib_pos_tokens_bwd {tag}")
        for n, t in dm.tensors().items():
            out[f"mlp_{tag}_{n}"] = _np(t)

    # attention: forward (plain, masked, gated), backward in both forms
    for M, s, B, HW in ((32, 16, 1, 64), (96, 48, 1, 192)):
        w = I.get_workload("w32" if M == 32 else "w96train", batch=B)
        inp = I.make_layer_inputs(w, 0, strong=True)
        mlp = R.PositionMLP.from_params(inp["freqs"], inp["mlp_q"], inp["mlp_k"], w.heads, 16)
        _, _, q16, k16 = R.rib_pos_tokens(mlp, M)
        qkv, dout = inp["qkv"].cuda(), inp["dout"].cuda()
        o, lse = R.rib_window_attn_fwd(qkv, M, s, q16, k16)
        done(f"rib_window_attn_fwd M={M}")
        out[f"out_{M}"], out[f"lse_{M}"] = _np(o), _np(lse)
        om, lm = R.rib_window_attn_fwd(qkv, M, s, q16, k16, region_mask=True)
        done(f"rib_window_attn_fwd_masked M={M}")
        out[f"out_masked_{M}"] = _np(om)
        for form, which in (("item", _abi.RIB_BWD_PER_ITEM), ("persist", _abi.RIB_BWD_PERSISTENT)):
            R.rib_set_bwd_kernel(which)
            g = R.rib_window_attn_bwd(qkv, o, dout, lse, M, s, q16, k16, mlp=mlp)
            done(f"rib_window_attn_bwd {form} M={M}")
            out[f"dkv_{form}_{M}"] = _np(g["dqkv"][:, :, :, 1:])
            out[f"dkp_{form}_{M}"] = _np(g["dkp"])
            out[f"~dq_{form}_{M}"] = _np(g["dqkv"][:, :, :, 0])
            out[f"~dqp_{form}_{M}"] = _np(g["dqp"])
            gm = R.rib_window_attn_bwd(qkv, om, dout, lm, M, s, q16, k16, region_mask=True)
            done(f"rib_window_attn_bwd_masked {form} M={M}")
            out[f"dkv_masked_{form}_{M}"] = _np(gm["dqkv"][:, :, :, 1:])
        R.rib_set_bwd_kernel(_abi.RIB_BWD_AUTO)

    # the fp32 forward on the tf32 tensor cores
    q32 = I.make_qkv(1, 64, 64, 3, 32, seed=4, dtype=torch.float32).cuda()
    mlp = R.PositionMLP.from_params(I.default_freqs(16), I.make_mlp(16, 64, 3, 16, 4, 0),
                                    I.make_mlp(16, 64, 3, 16, 4, 1), 3, 16)
    qp, kp, _, _ = R.rib_pos_tokens(mlp, 16)
    o32, l32 = R.rib_window_attn_fwd_tf32(q32, 16, 8, qp, kp)
    done("rib_window_attn_fwd_tf32")
    out["out_tf32"], out["lse_tf32"] = _np(o32), _np(l32)

    # convolutional local attention: gate, gated forward, backward
    B, H, W, C = 1, 32, 48, 192
    p = I.make_cla(C, 9)
    cla = R.ClaGate.from_params(p.w_dw, p.b_dw, p.w_pw, p.b_pw)
    x = I.make_features(B, H, W, C, 9).cuda()
    gate = R.rib_cla_gate(x, cla)
    done("rib_cla_gate")
    out["gate"] = _np(gate)
    qkv = I.make_qkv(B, H, W, 6, 32, seed=9).cuda()
    mlp = R.PositionMLP.from_params(I.default_freqs(16), I.make_mlp(16, 128, 6, 16, 9, 0),
                                    I.make_mlp(16, 128, 6, 16, 9, 1), 6, 16)
    _, _, q16, k16 = R.rib_pos_tokens(mlp, 16)
    o, og, lse = R.rib_window_attn_fwd_cla(qkv, 16, 8, gate, q16, k16)
    done("rib_window_attn_fwd_cla")
    out["out_gated"] = _np(og)
    dog = I.make_features(B, H, W, C, 10).cuda()
    gc = R.rib_cla_bwd(x, cla, gate, o.view(B, H, W, C), dog)
    done("rib_cla_bwd")
    for k in ("dout", "dx", "dw_dw", "db_dw", "dw_pw", "db_pw"):
        out[f"cla_{k}"] = _np(gc[k])

    # window gather / scatter and the allocation-free MLP backward
    xm = I.make_features(2, 32, 48, 24, 11).cuda()
    xw = R.rib_window_gather(xm, 16, 8)
    back = R.rib_window_scatter(xw, 32, 48, 16, 8)
    done("rib_window_gather / rib_window_scatter")
    out["gathered"], out["scattered"] = _np(xw), _np(back)
    mlp = R.PositionMLP.from_params(I.default_freqs(16), I.make_mlp(16, 128, 6, 16, 12, 0),
                                    I.make_mlp(16, 128, 6, 16, 12, 1), 6, 16)
    gq = I.randn((6, 32, 32, 16), seed=12, tag=7).cuda()
    gk = I.randn((6, 32, 32, 16), seed=12, tag=8).cuda()
    dm = R.PositionMLPGrad.empty_like(mlp)
    R.rib_pos_tokens_bwd_noalloc(mlp, 32, gq, gk, dm)
    done("rib_pos_tokens_bwd_noalloc")
    for n, t in dm.tensors().items():
        out[f"noalloc_{n}"] = _np(t)

    out["_debug_build"] = np.array([R.library().rib_debug_build()])
    np.savez(path, **out)
    print(f"{len(calls)} calls, status RIB_OK after each")


if __name__ == "__main__":
    main(sys.argv[1])
