"""The allocation-free position-MLP backward (rib_pos_tokens_bwd_noalloc).

Some callers cannot allocate device memory at the moment they need the MLP
gradients: code running while a CUDA graph is captured, hosts whose allocator
owns all device memory, or loops that cannot afford the synchronisation of a
cudaMalloc/cudaFree pair.  This entry point serves them with a scratch array
compiled into the library.  The test calls it through the C ABI twice in a
row, on different inputs, and checks each result against the fp64 oracle's
MLP backward and against the workspace-based rib_pos_tokens_bwd, with the
same bound the other MLP-backward tests use.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import rib_inputs as I
import windowed_attention_implicit_b200 as R
from windowed_attention_implicit_b200 import _abi

pytestmark = pytest.mark.gpu

MLP_REL = 1e-4


def _grads_via_abi(mlp, M, dqp, dkp):
    lib = R.library()
    out = R.PositionMLPGrad.empty_like(mlp)
    c, cg = mlp.c_struct(), out.c_struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.rib_pos_tokens_bwd_noalloc(ctypes.byref(c), M, dqp.data_ptr(), dkp.data_ptr(),
                                        ctypes.byref(cg), stream)
    assert rc == _abi.RIB_OK, R.rib_status_string(rc)
    return out


@pytest.mark.parametrize("M,hid", [(32, 128), (96, 128)])
def test_noalloc_matches_workspace_version_twice(M, hid):
    heads, rank, F = 6, 16, 16
    freqs = I.default_freqs(F)
    mq = I.make_mlp(F, hid, heads, rank, 41, 0, strong=True)
    mk = I.make_mlp(F, hid, heads, rank, 41, 1, strong=True)
    mlp = R.PositionMLP.from_params(freqs, mq, mk, heads, rank)
    for call in range(2):        # the shared scratch keeps the previous call's bytes
        gq = I.randn((heads, M, M, rank), seed=100 + call, tag=7).cuda()
        gk = I.randn((heads, M, M, rank), seed=200 + call, tag=8).cuda()
        got = _grads_via_abi(mlp, M, gq, gk)
        ref = R.rib_pos_tokens_bwd(mlp, M, gq, gk)
        torch.cuda.synchronize()
        assert R.rib_last_status()[0] == 0
        rq, rk = O.pos_tokens_backward(freqs, mq, mk, M, gq.double().cpu().numpy(),
                                       gk.double().cpu().numpy())
        exact = dict(zip(("q_dw1", "q_db1", "q_dw2", "q_db2"), rq))
        exact.update(zip(("k_dw1", "k_db1", "k_dw2", "k_db2"), rk))
        for name, e in exact.items():
            a = getattr(got, name).double().cpu().numpy()
            b = getattr(ref, name).double().cpu().numpy()
            rel = np.abs(a - e).max() / np.abs(e).max()
            assert rel <= MLP_REL, f"call {call} {name} vs oracle: rel {rel:.3e}"
            rel = np.abs(a - b).max() / max(np.abs(b).max(), 1e-30)
            assert rel <= MLP_REL, f"call {call} {name} vs workspace call: rel {rel:.3e}"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    heads, rank, F, hid, M = 6, 16, 16, 128, 128      # needs ~40 MiB of partials
    mlp = R.PositionMLP.from_params(I.default_freqs(F), I.make_mlp(F, hid, heads, rank, 1, 0),
                                    I.make_mlp(F, hid, heads, rank, 1, 1), heads, rank)
    assert R.rib_pos_tokens_bwd_workspace(mlp, M) > _abi.RIB_NOALLOC_SCRATCH_BYTES
    g = torch.zeros((heads, M, M, rank), device="cuda")
    out = R.PositionMLPGrad.empty_like(mlp)
    c, cg = mlp.c_struct(), out.c_struct()
    rc = R.library().rib_pos_tokens_bwd_noalloc(ctypes.byref(c), M, g.data_ptr(), g.data_ptr(),
                                                ctypes.byref(cg), None)
    assert rc == _abi.RIB_ERR_WORKSPACE
