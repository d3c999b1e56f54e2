"""CPU checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

import windowed_attention_implicit_b200 as R
from windowed_attention_implicit_b200 import _abi

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "rib.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rib_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("rib_pos_tokens", "rib_window_attn_fwd", "rib_window_attn_bwd",
              "rib_window_attn_bwd_workspace", "rib_last_status", "rib_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = R.library()
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _abi._SIGS, f"{name} has no ctypes signature"


def test_debug_library_exports_the_same_symbols_and_says_so():
    """librib_debug.so (the bounds-checked build) offers every declared entry
    point too; each library reports which build it is (no GPU call)."""
    import ctypes
    from windowed_attention_implicit_b200 import build as B
    if not os.path.exists(B.LIB_DEBUG):
        B.build(debug=True)
    dbg = ctypes.CDLL(B.LIB_DEBUG)
    for name in declared_functions():
        assert hasattr(dbg, name), name
    assert dbg.rib_debug_build() == 1
    assert R.library().rib_debug_build() == 0


def test_status_strings():
    lib = R.library()
    for code, name in ((0, "RIB_OK"), (-1, "RIB_ERR_ARG"), (-2, "RIB_ERR_SHAPE"),
                       (-3, "RIB_ERR_UNSUPPORTED"), (-4, "RIB_ERR_WORKSPACE"),
                       (-5, "RIB_ERR_CUDA"), (-6, "RIB_ERR_TIMEOUT"), (-7, "RIB_ERR_ALIGN"),
                       (-8, "RIB_ERR_BOUNDS")):
        assert lib.rib_status_string(code).decode() == name
    assert R.rib_version().startswith("rib-b200")


FAKE = 1 << 20        # 16-byte-aligned non-null stand-in; never dereferenced


def fwd(**kw):
    a = dict(qkv=FAKE, B=1, H=64, W=64, heads=2, d=32, M=16, s=0, qp=FAKE, kp=FAKE, r=16,
             scale=0.0, out=FAKE, lse=FAKE)
    a.update(kw)
    return R.library().rib_window_attn_fwd(
        a["qkv"], a["B"], a["H"], a["W"], a["heads"], a["d"], a["M"], a["s"], a["qp"],
        a["kp"], a["r"], a["scale"], a["out"], a["lse"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(qkv=None), _abi.RIB_ERR_ARG),
    (dict(B=-1), _abi.RIB_ERR_ARG),
    (dict(H=0), _abi.RIB_ERR_ARG),
    (dict(B=0, H=72), _abi.RIB_ERR_SHAPE),           # an empty batch is still shape-checked
    (dict(H=72), _abi.RIB_ERR_SHAPE),
    (dict(W=40), _abi.RIB_ERR_SHAPE),
    (dict(s=16), _abi.RIB_ERR_SHAPE),
    (dict(s=-8), _abi.RIB_ERR_SHAPE),
    (dict(d=64), _abi.RIB_ERR_UNSUPPORTED),
    (dict(r=8), _abi.RIB_ERR_UNSUPPORTED),
    (dict(M=8, H=64, W=64), _abi.RIB_ERR_UNSUPPORTED),
    (dict(s=4), _abi.RIB_ERR_UNSUPPORTED),
    (dict(qp=None), _abi.RIB_ERR_ARG),
    (dict(out=FAKE + 8), _abi.RIB_ERR_ALIGN),
    (dict(scale=float("nan")), _abi.RIB_ERR_ARG),
])
def test_fwd_validation(kw, code):
    assert fwd(**kw) == code


def test_empty_batch_is_a_no_op():
    # B = 0: valid shapes return RIB_OK before any pointer is looked at or
    # anything is launched (empty tensors may have null data pointers)
    assert fwd(B=0, qkv=None, out=None, lse=None, qp=None, kp=None) == _abi.RIB_OK
    lib = R.library()
    assert lib.rib_window_gather(None, 0, 64, 64, 96, 2, 16, 8, None, None) == _abi.RIB_OK
    assert lib.rib_window_scatter(None, 0, 64, 64, 96, 2, 16, 8, None, None) == _abi.RIB_OK
    assert lib.rib_cla_gate(None, 0, 16, 32, 96, FAKE, FAKE, FAKE, FAKE, None, None) == _abi.RIB_OK
    assert lib.rib_cla_gate(None, -1, 16, 32, 96, FAKE, FAKE, FAKE, FAKE, None, None) == _abi.RIB_ERR_ARG


def test_fwd_rank0_needs_no_position_tokens():
    # rank 0 with null Qp/Kp passes validation; stop it at the alignment check
    assert fwd(r=0, qp=None, kp=None, lse=FAKE + 4) == _abi.RIB_ERR_ALIGN


def test_bwd_workspace_sizes():
    ws = R.rib_window_attn_bwd_workspace
    B, H, W, h = 4, 192, 192, 6
    pix = B * h * H * W
    a = lambda x: (x + 255) // 256 * 256
    expect = a(pix * 4) * 2 + a(pix * 48 * 4) + a(pix * 16 * 4)
    assert ws(B, H, W, h, 32, 96, 16) == expect
    assert ws(B, H, W, h, 32, 96, 0) == a(pix * 4) * 2 + a(pix * 48 * 4)
    assert ws(B, H, W, h, 64, 96, 16) == 0          # unsupported -> 0
    assert ws(B, 100, W, h, 32, 96, 16) == 0        # bad shape -> 0


def test_bwd_validation():
    lib = R.library()
    def call(ws_bytes=1 << 40, **kw):
        a = dict(M=16, s=0, r=16, d=32, dqp=FAKE, ws=FAKE * 256)
        a.update(kw)
        return lib.rib_window_attn_bwd(FAKE, FAKE, FAKE, FAKE, 1, 64, 64, 2, a["d"], a["M"],
                                       a["s"], FAKE, FAKE, a["r"], 0.0, FAKE, a["dqp"], FAKE,
                                       None, None, a["ws"], ws_bytes, None)
    assert call(ws_bytes=16) == _abi.RIB_ERR_WORKSPACE
    assert call(ws=None) == _abi.RIB_ERR_WORKSPACE
    assert call(dqp=None) == _abi.RIB_ERR_ARG
    assert call(M=24) == _abi.RIB_ERR_SHAPE
    assert call(d=16) == _abi.RIB_ERR_UNSUPPORTED
    assert call(ws=FAKE * 256 + 16) == _abi.RIB_ERR_ALIGN


def test_gather_validation():
    lib = R.library()
    g = lambda **kw: lib.rib_window_gather(
        kw.get("x", FAKE), 1, kw.get("H", 64), kw.get("W", 64), kw.get("C", 8), kw.get("eb", 2),
        kw.get("M", 16), kw.get("s", 0), FAKE, None)
    assert g(x=None) == _abi.RIB_ERR_ARG
    assert g(eb=3) == _abi.RIB_ERR_ARG
    assert g(H=40) == _abi.RIB_ERR_SHAPE
    assert g(C=4) == _abi.RIB_ERR_UNSUPPORTED        # 8 bytes per pixel row
    assert g(s=4) == _abi.RIB_ERR_UNSUPPORTED
    assert g(M=12, H=48, W=48) == _abi.RIB_ERR_UNSUPPORTED


def test_pos_tokens_validation():
    lib = R.library()
    m = _abi.rib_mlp_t(16, FAKE, 64, 3, 16, *([FAKE] * 8))
    assert lib.rib_pos_tokens(None, 16, FAKE, FAKE, None, None, None) == _abi.RIB_ERR_ARG
    assert lib.rib_pos_tokens(ctypes.byref(m), 0, FAKE, FAKE, None, None, None) == _abi.RIB_ERR_ARG
    assert lib.rib_pos_tokens(ctypes.byref(m), 16, None, FAKE, None, None, None) == _abi.RIB_ERR_ARG
    m.n_freq = 0
    assert lib.rib_pos_tokens(ctypes.byref(m), 16, FAKE, FAKE, None, None, None) == _abi.RIB_ERR_ARG


def fwd_masked(**kw):
    a = dict(qkv=FAKE, B=1, H=64, W=64, heads=2, d=32, M=16, s=8, qp=FAKE, kp=FAKE, r=16,
             scale=0.0, out=FAKE, lse=FAKE)
    a.update(kw)
    return R.library().rib_window_attn_fwd_masked(
        a["qkv"], a["B"], a["H"], a["W"], a["heads"], a["d"], a["M"], a["s"], a["qp"],
        a["kp"], a["r"], a["scale"], a["out"], a["lse"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(qkv=None), _abi.RIB_ERR_ARG),
    (dict(H=72), _abi.RIB_ERR_SHAPE),
    (dict(s=16), _abi.RIB_ERR_SHAPE),
    (dict(s=4), _abi.RIB_ERR_UNSUPPORTED),
    (dict(d=64), _abi.RIB_ERR_UNSUPPORTED),
    (dict(qp=None), _abi.RIB_ERR_ARG),
    (dict(lse=FAKE + 4), _abi.RIB_ERR_ALIGN),
    (dict(scale=float("inf")), _abi.RIB_ERR_ARG),
    (dict(B=0, qkv=None, out=None, lse=None, qp=None, kp=None), _abi.RIB_OK),
])
def test_fwd_masked_validation(kw, code):
    assert fwd_masked(**kw) == code


def fwd_cla(**kw):
    a = dict(B=1, H=64, M=16, gate=FAKE, out=FAKE, out_gated=FAKE)
    a.update(kw)
    return R.library().rib_window_attn_fwd_cla(
        FAKE, a["B"], a["H"], 64, 2, 32, a["M"], 0, FAKE, FAKE, 16, 0.0, a["gate"], a["out"],
        a["out_gated"], FAKE, None)


def test_fwd_cla_validation():
    assert fwd_cla(gate=None) == _abi.RIB_ERR_ARG
    assert fwd_cla(out_gated=None) == _abi.RIB_ERR_ARG
    assert fwd_cla(gate=FAKE + 8) == _abi.RIB_ERR_ALIGN
    assert fwd_cla(out_gated=FAKE + 2) == _abi.RIB_ERR_ALIGN
    assert fwd_cla(H=72) == _abi.RIB_ERR_SHAPE
    assert fwd_cla(out=None) == _abi.RIB_ERR_ARG


def cla_gate(**kw):
    a = dict(x=FAKE, B=1, H=16, W=32, C=96, w_dw=FAKE, b_dw=FAKE, w_pw=FAKE, b_pw=FAKE,
             gate=FAKE)
    a.update(kw)
    return R.library().rib_cla_gate(a["x"], a["B"], a["H"], a["W"], a["C"], a["w_dw"],
                                    a["b_dw"], a["w_pw"], a["b_pw"], a["gate"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(H=0), _abi.RIB_ERR_ARG),
    (dict(C=-32), _abi.RIB_ERR_ARG),
    (dict(C=48), _abi.RIB_ERR_UNSUPPORTED),       # channels in multiples of 32
    (dict(H=12), _abi.RIB_ERR_SHAPE),             # tiles of 8 rows
    (dict(W=24), _abi.RIB_ERR_SHAPE),             # and 16 columns
    (dict(x=None), _abi.RIB_ERR_ARG),
    (dict(b_pw=None), _abi.RIB_ERR_ARG),
    (dict(gate=None), _abi.RIB_ERR_ARG),
    (dict(x=FAKE + 8), _abi.RIB_ERR_ALIGN),
    (dict(gate=FAKE + 8), _abi.RIB_ERR_ALIGN),
    (dict(w_pw=FAKE + 4), _abi.RIB_ERR_ALIGN),
    (dict(w_dw=FAKE + 2), _abi.RIB_ERR_ALIGN),
    (dict(B=0, H=12), _abi.RIB_ERR_SHAPE),        # an empty batch is still shape-checked
])
def test_cla_gate_validation(kw, code):
    assert cla_gate(**kw) == code


def test_cla_bwd_validation():
    lib = R.library()

    def call(**kw):
        a = dict(x=FAKE, B=1, H=16, W=32, C=96, w_dw=FAKE, b_dw=FAKE, w_pw=FAKE, gate=FAKE,
                 out=FAKE, dog=FAKE, do=FAKE, dx=FAKE, dw_dw=FAKE, db_dw=FAKE, dw_pw=FAKE,
                 db_pw=FAKE, ws=FAKE * 256, wsb=1 << 40)
        a.update(kw)
        return lib.rib_cla_bwd(a["x"], a["B"], a["H"], a["W"], a["C"], a["w_dw"], a["b_dw"],
                               a["w_pw"], a["gate"], a["out"], a["dog"], a["do"], a["dx"],
                               a["dw_dw"], a["db_dw"], a["dw_pw"], a["db_pw"], a["ws"],
                               a["wsb"], None)
    assert call(C=40) == _abi.RIB_ERR_UNSUPPORTED
    assert call(W=40) == _abi.RIB_ERR_SHAPE
    assert call(B=-1) == _abi.RIB_ERR_ARG
    assert call(dw_pw=None) == _abi.RIB_ERR_ARG
    assert call(B=0, dw_dw=None) == _abi.RIB_ERR_ARG
    assert call(dog=None) == _abi.RIB_ERR_ARG
    assert call(dx=None) == _abi.RIB_ERR_ARG
    assert call(out=FAKE + 8) == _abi.RIB_ERR_ALIGN
    assert call(dw_pw=FAKE + 4) == _abi.RIB_ERR_ALIGN
    assert call(db_pw=FAKE + 2) == _abi.RIB_ERR_ALIGN
    assert lib.rib_cla_bwd_workspace(1, 12, 32, 96) == 0    # bad shape -> 0
    assert lib.rib_cla_bwd_workspace(1, 16, 32, 40) == 0    # unsupported -> 0


def test_bwd_masked_validation():
    lib = R.library()

    def call(ws_bytes=1 << 40, **kw):
        a = dict(M=16, s=8, r=16, d=32, dqp=FAKE, ws=FAKE * 256)
        a.update(kw)
        return lib.rib_window_attn_bwd_masked(FAKE, FAKE, FAKE, FAKE, 1, 64, 64, 2, a["d"],
                                              a["M"], a["s"], FAKE, FAKE, a["r"], 0.0, FAKE,
                                              a["dqp"], FAKE, None, None, a["ws"], ws_bytes,
                                              None)
    assert call(ws_bytes=16) == _abi.RIB_ERR_WORKSPACE
    assert call(dqp=None) == _abi.RIB_ERR_ARG
    assert call(M=24) == _abi.RIB_ERR_SHAPE
    assert call(s=4) == _abi.RIB_ERR_UNSUPPORTED
    assert call(d=16) == _abi.RIB_ERR_UNSUPPORTED
    assert call(ws=FAKE * 256 + 16) == _abi.RIB_ERR_ALIGN


def test_work_entry_points_run_inside_nvtx_ranges(monkeypatch):
    log = []
    monkeypatch.setattr(R, "_nvtx_calls",
                        lambda: (lambda n: log.append(("push", n)), lambda: log.append("pop")))

    class FakeLib:
        pass
    fake = FakeLib()
    for name in _abi._SIGS:
        setattr(fake, name, (lambda n: (lambda *a: (n, a)))(name))

    def boom(*a):
        raise ValueError("from the library")
    fake.rib_window_scatter = boom
    lib = R._RangedLibrary(fake)
    assert lib.rib_window_attn_fwd(1, 2) == ("rib_window_attn_fwd", (1, 2))
    assert log == [("push", "rib_window_attn_fwd"), "pop"]
    log.clear()
    for quiet in ("rib_window_attn_bwd_workspace", "rib_cla_bwd_workspace", "rib_status_string",
                  "rib_last_status", "rib_trace_collect"):
        getattr(lib, quiet)()
    assert log == []
    with pytest.raises(ValueError):
        lib.rib_window_scatter()
    assert log == [("push", "rib_window_scatter"), "pop"]
    # the real library: the wrapped entry points keep their names
    assert R.library().rib_cla_bwd.__name__ == "rib_cla_bwd"


def test_backward_form_dispatch_by_window_and_override():
    """Windows up to 64 x 64 take the persistent backward, larger ones the
    per-item kernel; a forced form applies to every window until reset."""
    lib = R.library()
    assert lib.rib_bwd_kernel_for(16) == _abi.RIB_BWD_PERSISTENT
    assert lib.rib_bwd_kernel_for(64) == _abi.RIB_BWD_PERSISTENT
    assert lib.rib_bwd_kernel_for(96) == _abi.RIB_BWD_PER_ITEM
    assert lib.rib_bwd_kernel_for(256) == _abi.RIB_BWD_PER_ITEM
    try:
        R.rib_set_bwd_kernel(_abi.RIB_BWD_PER_ITEM)
        assert R.rib_bwd_kernel_for(16) == _abi.RIB_BWD_PER_ITEM
        R.rib_set_bwd_kernel(_abi.RIB_BWD_PERSISTENT)
        assert R.rib_bwd_kernel_for(96) == _abi.RIB_BWD_PERSISTENT
        assert lib.rib_set_bwd_kernel(7) == _abi.RIB_ERR_ARG
        assert R.rib_bwd_kernel_for(96) == _abi.RIB_BWD_PERSISTENT   # unchanged by the refusal
    finally:
        R.rib_set_bwd_kernel(_abi.RIB_BWD_AUTO)
    assert R.rib_bwd_kernel_for(32) == _abi.RIB_BWD_PERSISTENT
