"""RIB windowed attention on B200 (sm_100a): Python binding of librib.so.

Every function here has the name of a C entry point of include/rib.h and only
marshals arguments: it checks devices / dtypes / contiguity, allocates
missing outputs with torch (PyTorch is the device-memory and stream
provider), passes raw pointers and the current CUDA stream, and raises
RibError on a non-zero status.  All arithmetic runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback.

"Rank-Factorized Implicit Neural Bias: Scaling Super-Resolution Transformer
with FlashAttention" (arXiv 2603.06738): position tokens from a Fourier-
feature MLP on window coordinates are concatenated with the content tokens so
that the positional bias Qp Kp^T comes out of the attention dot product.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Dict, Optional, Tuple

import torch

from . import _abi

__all__ = [
    "RibError", "PositionMLP", "PositionMLPGrad", "PosTokenCache", "rib_pos_tokens",
    "rib_pos_tokens_bwd", "rib_pos_tokens_bwd_workspace", "rib_pos_tokens_bwd_noalloc",
    "rib_window_attn_fwd", "rib_window_attn_fwd_tf32", "rib_window_attn_bwd",
    "rib_window_attn_bwd_workspace",
    "rib_window_gather", "rib_window_scatter", "rib_last_status", "rib_status_string",
    "rib_set_wait_limit_ns", "rib_set_bwd_kernel", "rib_bwd_kernel_for", "rib_debug_wait_timeout", "rib_version", "library",
    "rib_trace_enable", "rib_trace_collect", "rib_debug_exp2", "ClaGate", "rib_cla_gate",
    "rib_window_attn_fwd_cla", "rib_cla_bwd", "rib_cla_bwd_workspace",
]


class RibError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {rib_status_string(code)} ({code})")


# Entry points that enqueue GPU work get an NVTX range named after them, so a
# profiler's timeline (ncu --nvtx, Nsight Systems) shows which call launched
# which kernels.  Without a tool attached a range costs well under a
# microsecond; where torch has no NVTX support the ranges are left out.
_NO_RANGE = ("_workspace", "rib_status_string", "rib_last_status", "rib_version",
             "rib_set_wait_limit_ns", "rib_trace_enable", "rib_trace_collect")


def _nvtx_calls():
    try:
        torch.cuda.nvtx.range_push("rib")
        torch.cuda.nvtx.range_pop()
        return torch.cuda.nvtx.range_push, torch.cuda.nvtx.range_pop
    except Exception:  # pragma: no cover - a torch build without NVTX
        return None


class _RangedLibrary:
    """librib.so with every work-enqueuing entry point wrapped in an NVTX
    range; other attributes are the ctypes library's own."""

    def __init__(self, cdll: ctypes.CDLL):
        self._cdll = cdll
        calls = _nvtx_calls()
        for name in _abi._SIGS:
            fn = getattr(cdll, name)
            if calls is not None and not any(t in name for t in _NO_RANGE):
                fn = self._ranged(name, fn, *calls)
            setattr(self, name, fn)

    @staticmethod
    def _ranged(name, fn, push, pop):
        def call(*args):
            push(name)
            try:
                return fn(*args)
            finally:
                pop()
        call.__name__ = name
        return call

    def __getattr__(self, name):
        return getattr(self._cdll, name)


_ranged_lib: Optional[_RangedLibrary] = None


def library() -> _RangedLibrary:
    """The loaded librib.so (raises if it is missing)."""
    global _ranged_lib
    if _ranged_lib is None:
        _ranged_lib = _RangedLibrary(_abi.load())
    return _ranged_lib


def _check(code: int, where: str) -> None:
    if code != _abi.RIB_OK:
        raise RibError(code, where)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor") -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _sizes(where: str, dev, **buffers) -> None:
    """Buffers handed to the library must hold exactly the elements the call
    reads or writes, on the device of the call's other tensors: the library
    takes bare pointers and can check neither.  buffers: name=(tensor or
    None, element count).  The library launches on the current CUDA device,
    so the call's tensors must live there (torch.cuda.set_device)."""
    if dev is not None and dev.type == "cuda" and dev.index != torch.cuda.current_device():
        raise RibError(_abi.RIB_ERR_ARG, f"{where}: tensors are on {dev}, the current device "
                       f"is cuda:{torch.cuda.current_device()}")
    for name, (t, n) in buffers.items():
        if t is None:
            continue
        if t.numel() != n:
            raise RibError(_abi.RIB_ERR_ARG,
                           f"{where}: {name} holds {t.numel()} elements, the call needs {n}")
        if t.device != dev:
            raise RibError(_abi.RIB_ERR_ARG, f"{where}: {name} is on {t.device}, not {dev}")


def _grad_sizes(dmlp: Optional["PositionMLPGrad"], mlp: Optional["PositionMLP"]):
    """Each position-MLP gradient sized like its weight."""
    if dmlp is None or mlp is None:
        return {}
    return {f"dmlp.{n}": (getattr(dmlp, n), getattr(mlp, n[:2] + n[3:]).numel())
            for n in ("q_dw1", "q_db1", "q_dw2", "q_db2", "k_dw1", "k_db1", "k_dw2", "k_db2")}


def _cla_sizes(cla: "ClaGate", C: int):
    return {"w_dw": (cla.w_dw, 9 * C), "b_dw": (cla.b_dw, C), "w_pw": (cla.w_pw, C * C),
            "b_pw": (cla.b_pw, C)}


def rib_status_string(code: int) -> str:
    return library().rib_status_string(int(code)).decode()


def rib_version() -> str:
    return library().rib_version().decode()


# ---------------------------------------------------------------- MLP weights

@dataclass
class PositionMLP:
    """Device fp32 weights of the two position MLPs (Linear layout [out][in])."""
    freqs: torch.Tensor
    q_w1: torch.Tensor
    q_b1: torch.Tensor
    q_w2: torch.Tensor
    q_b2: torch.Tensor
    k_w1: torch.Tensor
    k_b1: torch.Tensor
    k_w2: torch.Tensor
    k_b2: torch.Tensor
    heads: int
    rank: int

    @property
    def n_freq(self) -> int:
        return self.freqs.numel()

    @property
    def hidden(self) -> int:
        return self.q_w1.shape[0]

    @classmethod
    def from_params(cls, freqs, mlp_q, mlp_k, heads, rank, device="cuda"):
        """From host tensors (anything with w1, b1, w2, b2)."""
        f = lambda t: t.detach().to(device=device, dtype=torch.float32).contiguous()
        return cls(f(freqs), f(mlp_q.w1), f(mlp_q.b1), f(mlp_q.w2), f(mlp_q.b2),
                   f(mlp_k.w1), f(mlp_k.b1), f(mlp_k.w2), f(mlp_k.b2), heads, rank)

    def c_struct(self) -> _abi.rib_mlp_t:
        p = lambda t, n: _ptr(t, torch.float32, n)
        return _abi.rib_mlp_t(
            self.n_freq, p(self.freqs, "freqs"), self.hidden, self.heads, self.rank,
            p(self.q_w1, "q_w1"), p(self.q_b1, "q_b1"), p(self.q_w2, "q_w2"),
            p(self.q_b2, "q_b2"), p(self.k_w1, "k_w1"), p(self.k_b1, "k_b1"),
            p(self.k_w2, "k_w2"), p(self.k_b2, "k_b2"))

    def tensors(self) -> Tuple[torch.Tensor, ...]:
        """Every tensor the position tokens depend on."""
        return (self.freqs, self.q_w1, self.q_b1, self.q_w2, self.q_b2,
                self.k_w1, self.k_b1, self.k_w2, self.k_b2)

    def key(self) -> Tuple[int, ...]:
        """Addresses of those tensors (which storage the tokens come from)."""
        return tuple(t.data_ptr() for t in self.tensors())

    def versions(self) -> Tuple[int, ...]:
        """Their in-place modification counters (an optimizer step that
        updates the weights in place moves them on)."""
        return tuple(_tensor_version(t) for t in self.tensors())


def _tensor_version(t: torch.Tensor) -> int:
    try:
        return t._version
    except RuntimeError:  # an inference-mode tensor carries no version counter
        return -1


@dataclass
class PositionMLPGrad:
    q_dw1: torch.Tensor
    q_db1: torch.Tensor
    q_dw2: torch.Tensor
    q_db2: torch.Tensor
    k_dw1: torch.Tensor
    k_db1: torch.Tensor
    k_dw2: torch.Tensor
    k_db2: torch.Tensor

    @classmethod
    def empty_like(cls, mlp: PositionMLP):
        e = torch.empty_like
        return cls(e(mlp.q_w1), e(mlp.q_b1), e(mlp.q_w2), e(mlp.q_b2),
                   e(mlp.k_w1), e(mlp.k_b1), e(mlp.k_w2), e(mlp.k_b2))

    def c_struct(self) -> _abi.rib_mlp_grad_t:
        return _abi.rib_mlp_grad_t(*[_ptr(getattr(self, n), torch.float32, n) for n in (
            "q_dw1", "q_db1", "q_dw2", "q_db2", "k_dw1", "k_db1", "k_dw2", "k_db2")])

    def tensors(self) -> Dict[str, torch.Tensor]:
        return dict(self.__dict__)


# ---------------------------------------------------------------- entry points

def rib_pos_tokens(mlp: PositionMLP, window: int, qp=None, kp=None, qp_bf16=None,
                   kp_bf16=None, stream=None, with_bf16: bool = True):
    """Qp, Kp fp32 [heads][M][M][rank] (+ bf16 copies) for one window size."""
    shape = (mlp.heads, window, window, mlp.rank)
    dev = mlp.freqs.device
    qp = torch.empty(shape, device=dev, dtype=torch.float32) if qp is None else qp
    kp = torch.empty(shape, device=dev, dtype=torch.float32) if kp is None else kp
    if with_bf16:
        qp_bf16 = torch.empty(shape, device=dev, dtype=torch.bfloat16) if qp_bf16 is None else qp_bf16
        kp_bf16 = torch.empty(shape, device=dev, dtype=torch.bfloat16) if kp_bf16 is None else kp_bf16
    n = mlp.heads * int(window) ** 2 * mlp.rank
    _sizes("rib_pos_tokens", dev, qp=(qp, n), kp=(kp, n), qp_bf16=(qp_bf16, n),
           kp_bf16=(kp_bf16, n))
    c = mlp.c_struct()
    _check(library().rib_pos_tokens(
        ctypes.byref(c), int(window), _ptr(qp, torch.float32, "qp"), _ptr(kp, torch.float32, "kp"),
        _ptr(qp_bf16, torch.bfloat16, "qp_bf16"), _ptr(kp_bf16, torch.bfloat16, "kp_bf16"),
        _stream(stream)), "rib_pos_tokens")
    return qp, kp, qp_bf16, kp_bf16


def rib_pos_tokens_bwd_workspace(mlp: PositionMLP, window: int) -> int:
    c = mlp.c_struct()
    return int(library().rib_pos_tokens_bwd_workspace(ctypes.byref(c), int(window)))


def rib_pos_tokens_bwd(mlp: PositionMLP, window: int, dqp: torch.Tensor, dkp: torch.Tensor,
                       dmlp: Optional["PositionMLPGrad"] = None, workspace=None, stream=None):
    """Position-MLP gradients from dL/dQp, dL/dKp ([heads][M][M][rank] fp32)."""
    dmlp = PositionMLPGrad.empty_like(mlp) if dmlp is None else dmlp
    n = mlp.heads * int(window) ** 2 * mlp.rank
    _sizes("rib_pos_tokens_bwd", mlp.freqs.device, dqp=(dqp, n), dkp=(dkp, n),
           **_grad_sizes(dmlp, mlp))
    need = rib_pos_tokens_bwd_workspace(mlp, window)
    if workspace is None:
        workspace = torch.empty(max(need, 256), device=dqp.device, dtype=torch.uint8)
    c, cg = mlp.c_struct(), dmlp.c_struct()
    _check(library().rib_pos_tokens_bwd(
        ctypes.byref(c), int(window), _ptr(dqp, torch.float32, "dqp"),
        _ptr(dkp, torch.float32, "dkp"), ctypes.byref(cg), _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)), "rib_pos_tokens_bwd")
    return dmlp


def rib_pos_tokens_bwd_noalloc(mlp: PositionMLP, window: int, dqp: torch.Tensor,
                               dkp: torch.Tensor, dmlp: "PositionMLPGrad", stream=None):
    """rib_pos_tokens_bwd for callers that cannot allocate device memory at
    the point of the call (inside CUDA graph capture, under an allocator that
    owns all device memory, or where cudaMalloc's synchronisation is too
    costly).  The library's own static 24 MiB device scratch is used instead
    of a workspace; `dmlp` must be given (preallocated).  Calls that overlap
    on the GPU share that scratch and race; the first call on a device should
    precede any stream capture."""
    n = mlp.heads * int(window) ** 2 * mlp.rank
    _sizes("rib_pos_tokens_bwd_noalloc", mlp.freqs.device, dqp=(dqp, n), dkp=(dkp, n),
           **_grad_sizes(dmlp, mlp))
    c, cg = mlp.c_struct(), dmlp.c_struct()
    _check(library().rib_pos_tokens_bwd_noalloc(
        ctypes.byref(c), int(window), _ptr(dqp, torch.float32, "dqp"),
        _ptr(dkp, torch.float32, "dkp"), ctypes.byref(cg), _stream(stream)),
        "rib_pos_tokens_bwd_noalloc")
    return dmlp


def rib_window_attn_fwd(qkv: torch.Tensor, window: int, shift: int, qp_bf16=None,
                        kp_bf16=None, rank: int = 16, scale: float = 0.0, out=None, lse=None,
                        stream=None, region_mask: bool = False):
    """out bf16 [B][H][W][heads][d], lse fp32 [B][heads][H][W].

    region_mask: the optional shifted-window region mask
    (rib_window_attn_fwd_masked)."""
    B, H, W, three, heads, d = qkv.shape
    if three != 3:
        raise ValueError("qkv must be [B][H][W][3][heads][head_dim]")
    out = torch.empty((B, H, W, heads, d), device=qkv.device, dtype=torch.bfloat16) if out is None else out
    lse = torch.empty((B, heads, H, W), device=qkv.device, dtype=torch.float32) if lse is None else lse
    name = "rib_window_attn_fwd_masked" if region_mask else "rib_window_attn_fwd"
    nt = heads * int(window) ** 2 * int(rank)
    _sizes(name, qkv.device, out=(out, B * H * W * heads * d), lse=(lse, B * heads * H * W),
           qp_bf16=(qp_bf16 if rank > 0 else None, nt),
           kp_bf16=(kp_bf16 if rank > 0 else None, nt))
    _check(getattr(library(), name)(
        _ptr(qkv, torch.bfloat16, "qkv"), B, H, W, heads, d, int(window), int(shift),
        _ptr(qp_bf16, torch.bfloat16, "qp_bf16"), _ptr(kp_bf16, torch.bfloat16, "kp_bf16"),
        int(rank), float(scale), _ptr(out, torch.bfloat16, "out"),
        _ptr(lse, torch.float32, "lse"), _stream(stream)), name)
    return out, lse


def rib_window_attn_fwd_tf32(qkv: torch.Tensor, window: int, shift: int, qp=None, kp=None,
                             rank: int = 16, scale: float = 0.0, out=None, lse=None,
                             stream=None):
    """fp32 forward on the tf32 tensor cores: qkv fp32 [B][H][W][3][heads][d],
    qp/kp fp32 [heads][M][M][rank]; returns out fp32 [B][H][W][heads][d] and
    lse fp32 [B][heads][H][W]."""
    B, H, W, three, heads, d = qkv.shape
    if three != 3:
        raise ValueError("qkv must be [B][H][W][3][heads][head_dim]")
    out = torch.empty((B, H, W, heads, d), device=qkv.device, dtype=torch.float32) if out is None else out
    lse = torch.empty((B, heads, H, W), device=qkv.device, dtype=torch.float32) if lse is None else lse
    nt = heads * int(window) ** 2 * int(rank)
    name = "rib_window_attn_fwd_tf32"
    _sizes(name, qkv.device, out=(out, B * H * W * heads * d), lse=(lse, B * heads * H * W),
           qp=(qp if rank > 0 else None, nt), kp=(kp if rank > 0 else None, nt))
    _check(library().rib_window_attn_fwd_tf32(
        _ptr(qkv, torch.float32, "qkv"), B, H, W, heads, d, int(window), int(shift),
        _ptr(qp, torch.float32, "qp"), _ptr(kp, torch.float32, "kp"), int(rank), float(scale),
        _ptr(out, torch.float32, "out"), _ptr(lse, torch.float32, "lse"), _stream(stream)), name)
    return out, lse


@dataclass
class ClaGate:
    """Device fp32 weights of the convolutional local attention gate:
    depth-wise 3x3 (w_dw [C][3][3], b_dw [C]) then point-wise 1x1
    (w_pw [C_out][C_in], b_pw [C]) then a sigmoid."""
    w_dw: torch.Tensor
    b_dw: torch.Tensor
    w_pw: torch.Tensor
    b_pw: torch.Tensor

    @classmethod
    def from_params(cls, w_dw, b_dw, w_pw, b_pw, device="cuda"):
        f = lambda t: torch.as_tensor(t).detach().to(device=device, dtype=torch.float32).contiguous()
        return cls(f(w_dw), f(b_dw), f(w_pw), f(b_pw))

    @property
    def channels(self) -> int:
        return self.b_dw.numel()


def rib_cla_gate(x: torch.Tensor, cla: ClaGate, gate=None, stream=None) -> torch.Tensor:
    """G bf16 [B][H][W][C] = sigmoid(PW1x1(DW3x3(x))) for x bf16 [B][H][W][C]."""
    B, H, W, C = x.shape
    gate = torch.empty_like(x) if gate is None else gate
    _sizes("rib_cla_gate", x.device, gate=(gate, x.numel()), **_cla_sizes(cla, C))
    f32 = torch.float32
    _check(library().rib_cla_gate(
        _ptr(x, torch.bfloat16, "x"), B, H, W, C, _ptr(cla.w_dw, f32, "w_dw"),
        _ptr(cla.b_dw, f32, "b_dw"), _ptr(cla.w_pw, f32, "w_pw"), _ptr(cla.b_pw, f32, "b_pw"),
        _ptr(gate, torch.bfloat16, "gate"), _stream(stream)), "rib_cla_gate")
    return gate


def rib_window_attn_fwd_cla(qkv: torch.Tensor, window: int, shift: int, gate: torch.Tensor,
                            qp_bf16=None, kp_bf16=None, rank: int = 16, scale: float = 0.0,
                            out=None, out_gated=None, lse=None, stream=None):
    """(out, out_gated, lse): the attention output O, O * gate (gate bf16
    [B][H][W][heads*d]) and lse, from one forward launch."""
    B, H, W, three, heads, d = qkv.shape
    if three != 3:
        raise ValueError("qkv must be [B][H][W][3][heads][head_dim]")
    if tuple(gate.shape) not in ((B, H, W, heads * d), (B, H, W, heads, d)):
        raise ValueError("gate must be [B][H][W][heads*head_dim]")
    shape = (B, H, W, heads, d)
    out = torch.empty(shape, device=qkv.device, dtype=torch.bfloat16) if out is None else out
    out_gated = torch.empty(shape, device=qkv.device, dtype=torch.bfloat16) if out_gated is None else out_gated
    lse = torch.empty((B, heads, H, W), device=qkv.device, dtype=torch.float32) if lse is None else lse
    n_out, nt = B * H * W * heads * d, heads * int(window) ** 2 * int(rank)
    _sizes("rib_window_attn_fwd_cla", qkv.device, gate=(gate, n_out), out=(out, n_out),
           out_gated=(out_gated, n_out), lse=(lse, B * heads * H * W),
           qp_bf16=(qp_bf16 if rank > 0 else None, nt),
           kp_bf16=(kp_bf16 if rank > 0 else None, nt))
    _check(library().rib_window_attn_fwd_cla(
        _ptr(qkv, torch.bfloat16, "qkv"), B, H, W, heads, d, int(window), int(shift),
        _ptr(qp_bf16, torch.bfloat16, "qp_bf16"), _ptr(kp_bf16, torch.bfloat16, "kp_bf16"),
        int(rank), float(scale), _ptr(gate, torch.bfloat16, "gate"),
        _ptr(out, torch.bfloat16, "out"), _ptr(out_gated, torch.bfloat16, "out_gated"),
        _ptr(lse, torch.float32, "lse"), _stream(stream)), "rib_window_attn_fwd_cla")
    return out, out_gated, lse


def rib_cla_bwd_workspace(B: int, H: int, W: int, C: int) -> int:
    return int(library().rib_cla_bwd_workspace(B, H, W, C))


def rib_cla_bwd(x: torch.Tensor, cla: ClaGate, gate: torch.Tensor, out: torch.Tensor,
                dout_gated: torch.Tensor, dout=None, dx=None, workspace=None, stream=None):
    """Backward of O' = O * gate: returns dict(dout = dO' * G (the attention
    backward's input), dx, dw_dw, db_dw, dw_pw, db_pw).  out / dout_gated may be
    [B][H][W][heads][d] or [B][H][W][C]."""
    B, H, W, C = x.shape
    dev = x.device
    dout = torch.empty(out.shape, device=dev, dtype=torch.bfloat16) if dout is None else dout
    dx = torch.empty_like(x) if dx is None else dx
    g = {k: torch.empty_like(getattr(cla, k.replace("d", "", 1)))
         for k in ("dw_dw", "db_dw", "dw_pw", "db_pw")}
    n = x.numel()
    _sizes("rib_cla_bwd", dev, gate=(gate, n), out=(out, n), dout_gated=(dout_gated, n),
           dout=(dout, n), dx=(dx, n), **_cla_sizes(cla, C))
    need = rib_cla_bwd_workspace(B, H, W, C)
    if workspace is None:
        workspace = torch.empty(max(need, 256), device=dev, dtype=torch.uint8)
    bf, f32 = torch.bfloat16, torch.float32
    _check(library().rib_cla_bwd(
        _ptr(x, bf, "x"), B, H, W, C, _ptr(cla.w_dw, f32, "w_dw"), _ptr(cla.b_dw, f32, "b_dw"),
        _ptr(cla.w_pw, f32, "w_pw"), _ptr(gate, bf, "gate"), _ptr(out, bf, "out"),
        _ptr(dout_gated, bf, "dout_gated"), _ptr(dout, bf, "dout"), _ptr(dx, bf, "dx"),
        _ptr(g["dw_dw"], f32, "dw_dw"), _ptr(g["db_dw"], f32, "db_dw"),
        _ptr(g["dw_pw"], f32, "dw_pw"), _ptr(g["db_pw"], f32, "db_pw"),
        _ptr(workspace, None, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream)), "rib_cla_bwd")
    return dict(dout=dout, dx=dx, **g)


def rib_window_attn_bwd_workspace(B, H, W, heads, head_dim, window, rank,
                                  mlp: Optional[PositionMLP] = None) -> int:
    c = mlp.c_struct() if mlp is not None else None
    return int(library().rib_window_attn_bwd_workspace(
        B, H, W, heads, head_dim, int(window), int(rank),
        ctypes.byref(c) if c is not None else None))


def rib_window_attn_bwd(qkv, out, dout, lse, window: int, shift: int, qp_bf16=None,
                        kp_bf16=None, rank: int = 16, scale: float = 0.0,
                        mlp: Optional[PositionMLP] = None, dqkv=None, dqp=None, dkp=None,
                        dmlp: Optional[PositionMLPGrad] = None, workspace=None, stream=None,
                        region_mask: bool = False):
    """Returns dict(dqkv, dqp, dkp, dmlp).  dmlp is computed when mlp is given.
    region_mask: as for rib_window_attn_fwd (rib_window_attn_bwd_masked)."""
    B, H, W, _, heads, d = qkv.shape
    dev = qkv.device
    dqkv = torch.empty_like(qkv) if dqkv is None else dqkv
    if rank > 0:
        pshape = (heads, window, window, rank)
        dqp = torch.empty(pshape, device=dev, dtype=torch.float32) if dqp is None else dqp
        dkp = torch.empty(pshape, device=dev, dtype=torch.float32) if dkp is None else dkp
    if mlp is not None and dmlp is None:
        dmlp = PositionMLPGrad.empty_like(mlp)
    name = "rib_window_attn_bwd_masked" if region_mask else "rib_window_attn_bwd"
    n_out, nt = B * H * W * heads * d, heads * int(window) ** 2 * int(rank)
    pos = rank > 0
    _sizes(name, dev, out=(out, n_out), dout=(dout, n_out), lse=(lse, B * heads * H * W),
           dqkv=(dqkv, qkv.numel()), qp_bf16=(qp_bf16 if pos else None, nt),
           kp_bf16=(kp_bf16 if pos else None, nt), dqp=(dqp if pos else None, nt),
           dkp=(dkp if pos else None, nt), **_grad_sizes(dmlp, mlp))
    need = rib_window_attn_bwd_workspace(B, H, W, heads, d, window, rank, mlp)
    if workspace is None:
        workspace = torch.empty(max(need, 256), device=dev, dtype=torch.uint8)
    c_mlp = mlp.c_struct() if mlp is not None else None
    c_dmlp = dmlp.c_struct() if (mlp is not None and dmlp is not None) else None
    _check(getattr(library(), name)(
        _ptr(qkv, torch.bfloat16, "qkv"), _ptr(out, torch.bfloat16, "out"),
        _ptr(dout, torch.bfloat16, "dout"), _ptr(lse, torch.float32, "lse"),
        B, H, W, heads, d, int(window), int(shift),
        _ptr(qp_bf16, torch.bfloat16, "qp_bf16"), _ptr(kp_bf16, torch.bfloat16, "kp_bf16"),
        int(rank), float(scale), _ptr(dqkv, torch.bfloat16, "dqkv"),
        _ptr(dqp, torch.float32, "dqp"), _ptr(dkp, torch.float32, "dkp"),
        ctypes.byref(c_mlp) if c_mlp is not None else None,
        ctypes.byref(c_dmlp) if c_dmlp is not None else None,
        _ptr(workspace, None, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream)), name)
    return {"dqkv": dqkv, "dqp": dqp, "dkp": dkp, "dmlp": dmlp}


def rib_window_gather(x: torch.Tensor, window: int, shift: int, out=None, stream=None):
    """x [B][H][W][C] -> [B][nW][M*M][C] (roll by -shift, partition)."""
    B, H, W, C = x.shape
    nW = (H // window) * (W // window)
    out = torch.empty((B, nW, window * window, C), device=x.device, dtype=x.dtype) if out is None else out
    _sizes("rib_window_gather", x.device, out=(out, B * nW * window * window * C))
    _check(library().rib_window_gather(
        _ptr(x, None, "x"), B, H, W, C, x.element_size(), int(window), int(shift),
        _ptr(out, x.dtype, "out"), _stream(stream)), "rib_window_gather")
    return out


def rib_window_scatter(xw: torch.Tensor, H: int, W: int, window: int, shift: int, out=None,
                       stream=None):
    """Inverse of rib_window_gather."""
    B, nW, N, C = xw.shape
    out = torch.empty((B, H, W, C), device=xw.device, dtype=xw.dtype) if out is None else out
    _sizes("rib_window_scatter", xw.device, out=(out, B * H * W * C))
    if (window > 0 and H % window == 0 and W % window == 0 and
            (nW, N) != ((H // window) * (W // window), window * window)):
        raise RibError(_abi.RIB_ERR_ARG, f"rib_window_scatter: xw is [B][{nW}][{N}][C], the "
                       f"{window}x{window} windows of a {H}x{W} map need "
                       f"[B][{(H // window) * (W // window)}][{window * window}][C]")
    _check(library().rib_window_scatter(
        _ptr(xw, None, "xw"), B, H, W, C, xw.element_size(), int(window), int(shift),
        _ptr(out, xw.dtype, "out"), _stream(stream)), "rib_window_scatter")
    return out


def rib_last_status() -> Tuple[int, int]:
    site = ctypes.c_int(0)
    code = library().rib_last_status(ctypes.byref(site))
    return int(code), int(site.value)


def rib_set_wait_limit_ns(limit_ns: int) -> None:
    _check(library().rib_set_wait_limit_ns(int(limit_ns)), "rib_set_wait_limit_ns")


def rib_set_bwd_kernel(which: int) -> None:
    """Form of the attention backward kernel, process-wide: _abi.RIB_BWD_AUTO
    (by window size), RIB_BWD_PER_ITEM or RIB_BWD_PERSISTENT."""
    _check(library().rib_set_bwd_kernel(int(which)), "rib_set_bwd_kernel")


def rib_bwd_kernel_for(window: int) -> int:
    """The backward form a call with this window size would use."""
    return int(library().rib_bwd_kernel_for(int(window)))


def rib_debug_exp2(x: torch.Tensor, stream=None) -> torch.Tensor:
    """2^x with the attention kernels' FMA-pipe exponential (test hook)."""
    y = torch.empty_like(x)
    _check(library().rib_debug_exp2(_ptr(x, torch.float32, "x"), _ptr(y, torch.float32, "y"),
                                    x.numel(), _stream(stream)), "rib_debug_exp2")
    return y


def rib_debug_wait_timeout(limit_ns: int, stream=None) -> None:
    _check(library().rib_debug_wait_timeout(int(limit_ns), _stream(stream)),
           "rib_debug_wait_timeout")


def rib_trace_enable(on: bool = True) -> None:
    _check(library().rib_trace_enable(1 if on else 0), "rib_trace_enable")


def rib_trace_collect() -> Dict[str, Tuple[int, float]]:
    """{kernel: (launches, total_ms)} of the launches traced since enabling."""
    entries = (_abi.rib_trace_entry_t * 32)()
    n = ctypes.c_int(0)
    _check(library().rib_trace_collect(ctypes.cast(entries, ctypes.c_void_p), 32,
                                       ctypes.byref(n)), "rib_trace_collect")
    return {entries[i].kernel.decode(): (int(entries[i].launches), float(entries[i].total_ms))
            for i in range(n.value)}


# ---------------------------------------------------------------- geometry cache

class PosTokenCache:
    """Qp/Kp per window geometry, computed once and reused across windows,
    batch entries and layers (they depend only on the geometry and the MLP).

    An entry is keyed by the window and the addresses of the MLP's tensors
    (frequencies, weights and biases), and holds references to them, so no
    other tensor can take those addresses while it lives.  It is recomputed
    when any of them has been modified in place since (an optimizer step),
    and replaced, not kept beside the new one."""

    def __init__(self):
        self._cache = {}

    def get(self, mlp: PositionMLP, window: int, stream=None):
        k = (mlp.key(), int(window))
        ver = mlp.versions()
        e = self._cache.get(k)
        if e is None or e[0] != ver:
            tokens = rib_pos_tokens(mlp, window, stream=stream)
            self._cache[k] = (ver, tokens, mlp.tensors())
            e = self._cache[k]
        return e[1]

    def clear(self):
        self._cache.clear()

    def __len__(self):
        return len(self._cache)
