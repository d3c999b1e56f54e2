"""ctypes view of librib.so (include/rib.h).  Loading only; no computation."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# RIB_DEBUG_LIBRARY=1 selects the bounds-checked debug build of the same
# library (librib_debug.so); otherwise the release build is loaded.
LIB_PATH = os.path.join(_HERE, "librib_debug.so" if os.environ.get("RIB_DEBUG_LIBRARY") == "1"
                        else "librib.so")

RIB_OK = 0
RIB_ERR_ARG = -1
RIB_ERR_SHAPE = -2
RIB_ERR_UNSUPPORTED = -3
RIB_ERR_WORKSPACE = -4
RIB_ERR_CUDA = -5
RIB_ERR_TIMEOUT = -6
RIB_ERR_ALIGN = -7
RIB_ERR_BOUNDS = -8
RIB_NOALLOC_SCRATCH_BYTES = 24 * 1024 * 1024
RIB_BWD_AUTO = 0
RIB_BWD_PER_ITEM = 1
RIB_BWD_PERSISTENT = 2

_p = ctypes.c_void_p
_fp = ctypes.POINTER(ctypes.c_float)
_i = ctypes.c_int


class rib_mlp_t(ctypes.Structure):
    _fields_ = [
        ("n_freq", _i), ("freqs", _p), ("d_hidden", _i), ("heads", _i), ("rank", _i),
        ("q_w1", _p), ("q_b1", _p), ("q_w2", _p), ("q_b2", _p),
        ("k_w1", _p), ("k_b1", _p), ("k_w2", _p), ("k_b2", _p),
    ]


class rib_trace_entry_t(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_char_p), ("launches", _i), ("total_ms", ctypes.c_double)]


class rib_mlp_grad_t(ctypes.Structure):
    _fields_ = [
        ("q_dw1", _p), ("q_db1", _p), ("q_dw2", _p), ("q_db2", _p),
        ("k_dw1", _p), ("k_db1", _p), ("k_dw2", _p), ("k_db2", _p),
    ]


_SIGS = {
    "rib_pos_tokens": (_i, [ctypes.POINTER(rib_mlp_t), _i, _p, _p, _p, _p, _p]),
    "rib_pos_tokens_bwd_workspace": (ctypes.c_size_t, [ctypes.POINTER(rib_mlp_t), _i]),
    "rib_pos_tokens_bwd": (_i, [ctypes.POINTER(rib_mlp_t), _i, _p, _p,
                                ctypes.POINTER(rib_mlp_grad_t), _p, ctypes.c_size_t, _p]),
    "rib_pos_tokens_bwd_noalloc": (_i, [ctypes.POINTER(rib_mlp_t), _i, _p, _p,
                                        ctypes.POINTER(rib_mlp_grad_t), _p]),
    "rib_window_attn_fwd": (_i, [_p, _i, _i, _i, _i, _i, _i, _i, _p, _p, _i,
                                 ctypes.c_float, _p, _p, _p]),
    "rib_window_attn_fwd_masked": (_i, [_p, _i, _i, _i, _i, _i, _i, _i, _p, _p, _i,
                                        ctypes.c_float, _p, _p, _p]),
    "rib_window_attn_fwd_cla": (_i, [_p, _i, _i, _i, _i, _i, _i, _i, _p, _p, _i,
                                     ctypes.c_float, _p, _p, _p, _p, _p]),
    "rib_window_attn_fwd_tf32": (_i, [_p, _i, _i, _i, _i, _i, _i, _i, _p, _p, _i,
                                      ctypes.c_float, _p, _p, _p]),
    "rib_cla_gate": (_i, [_p, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p]),
    "rib_cla_bwd_workspace": (ctypes.c_size_t, [_i, _i, _i, _i]),
    "rib_cla_bwd": (_i, [_p, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p,
                         _p, ctypes.c_size_t, _p]),
    "rib_window_attn_bwd_workspace": (ctypes.c_size_t,
                                      [_i, _i, _i, _i, _i, _i, _i,
                                       ctypes.POINTER(rib_mlp_t)]),
    "rib_window_attn_bwd": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p, _p,
                                 _i, ctypes.c_float, _p, _p, _p,
                                 ctypes.POINTER(rib_mlp_t),
                                 ctypes.POINTER(rib_mlp_grad_t), _p, ctypes.c_size_t, _p]),
    "rib_window_attn_bwd_masked": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p, _p,
                                        _i, ctypes.c_float, _p, _p, _p,
                                        ctypes.POINTER(rib_mlp_t),
                                        ctypes.POINTER(rib_mlp_grad_t), _p, ctypes.c_size_t,
                                        _p]),
    "rib_window_gather": (_i, [_p, _i, _i, _i, _i, _i, _i, _i, _p, _p]),
    "rib_window_scatter": (_i, [_p, _i, _i, _i, _i, _i, _i, _i, _p, _p]),
    "rib_status_string": (ctypes.c_char_p, [_i]),
    "rib_last_status": (_i, [ctypes.POINTER(_i)]),
    "rib_set_wait_limit_ns": (_i, [ctypes.c_ulonglong]),
    "rib_set_bwd_kernel": (_i, [_i]),
    "rib_bwd_kernel_for": (_i, [_i]),
    "rib_debug_wait_timeout": (_i, [ctypes.c_ulonglong, _p]),
    "rib_debug_exp2": (_i, [_p, _p, _i, _p]),
    "rib_debug_build": (_i, []),
    "rib_debug_guard_info": (_i, [ctypes.POINTER(ctypes.c_ulonglong)]),
    "rib_debug_guard_selftest": (_i, [_i, _i, _p]),
    "rib_version": (ctypes.c_char_p, []),
    "rib_trace_enable": (_i, [_i]),
    "rib_trace_collect": (_i, [ctypes.c_void_p, _i, ctypes.POINTER(_i)]),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads librib.so once.  Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(
            f"{os.path.basename(path)} not found at {path}; build it with "
            "`python -m windowed_attention_implicit_b200.build`"
            f"{' --debug' if path.endswith('_debug.so') else ''}")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
