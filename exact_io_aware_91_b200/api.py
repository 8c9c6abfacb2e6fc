"""Python binding of the C ABI in ``include/fa.h`` (argument marshalling only).

Every function here has the name of the C entry point it calls.  PyTorch provides
device memory and the current CUDA stream; all arithmetic happens in the CUDA
kernels of ``libfa_b200.so``.  There is no fallback: if the library is missing
or the device is not supported, the call raises.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

from . import build as _build

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_MISALIGNED = 3
FA_ERR_CUDA = 4
FA_ERR_TIMEOUT = 5
FA_ERR_RANGE = 6

EXPORTS = ("fa_fwd", "fa_fwd_gqa", "fa_fwd_workspace_size", "fa_fwd_ws", "fa_fwd_f32", "fa_bwd_workspace_size", "fa_bwd", "fa_bwd_gqa_workspace_size",
           "fa_bwd_gqa", "fa_bwd_ws_workspace_size", "fa_bwd_ws", "fa_attn_fwd_workspace_size", "fa_attn_fwd", "fa_attn_bwd_workspace_size", "fa_attn_bwd",
           "fa_attn_fwd_fp8_workspace_size", "fa_attn_fwd_fp8", "fa_bwd_noalloc", "fa_last_device_status",
           "fa_device_status", "fa_bwd_set_phase_events", "fa_selftest_wait_timeout", "fa_selftest_exp2",
           "fa_status_str")

# Size of the scratch array fa_bwd_noalloc uses instead of a caller workspace.
FA_BWD_NOALLOC_MAX_WORKSPACE = 64 << 20


class FaAttnProblem(ctypes.Structure):
    """``fa_attn_problem`` of ``include/fa.h``."""
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("H_kv", ctypes.c_int), ("N", ctypes.c_int),
                ("d", ctypes.c_int), ("scale", ctypes.c_float), ("causal", ctypes.c_int),
                ("window_left", ctypes.c_int), ("window_right", ctypes.c_int)]


class FAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {status_str(status)} ({status})")
        self.status = status


_LIB = None


def library() -> ctypes.CDLL:
    """Load ``libfa_b200.so`` from the package directory (raises if it is not built)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = _build.LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m exact_io_aware_91_b200.build` "
            "(there is no non-CUDA fallback)"
        )
    lib = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    lib.fa_fwd.restype = i
    lib.fa_fwd_gqa.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    lib.fa_fwd_gqa.restype = i
    lib.fa_fwd_workspace_size.argtypes = [i, i, i, i]
    lib.fa_fwd_workspace_size.restype = sz
    lib.fa_fwd_ws.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, sz, vp]
    lib.fa_fwd_ws.restype = i
    lib.fa_fwd_f32.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    lib.fa_fwd_f32.restype = i
    lib.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    lib.fa_bwd_workspace_size.restype = sz
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, vp]
    lib.fa_bwd.restype = i
    lib.fa_bwd_gqa_workspace_size.argtypes = [i, i, i, i, i]
    lib.fa_bwd_gqa_workspace_size.restype = sz
    lib.fa_bwd_gqa.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, sz, vp]
    lib.fa_bwd_gqa.restype = i
    lib.fa_bwd_ws_workspace_size.argtypes = [i, i, i, i, i]
    lib.fa_bwd_ws_workspace_size.restype = sz
    lib.fa_bwd_ws.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, sz, vp, sz, vp]
    lib.fa_bwd_ws.restype = i
    pp = ctypes.POINTER(FaAttnProblem)
    lib.fa_attn_fwd_workspace_size.argtypes = [pp]
    lib.fa_attn_fwd_workspace_size.restype = sz
    lib.fa_attn_fwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.fa_attn_fwd.restype = i
    lib.fa_attn_bwd_workspace_size.argtypes = [pp]
    lib.fa_attn_bwd_workspace_size.restype = sz
    lib.fa_attn_bwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.fa_attn_bwd.restype = i
    lib.fa_attn_fwd_fp8_workspace_size.argtypes = [pp]
    lib.fa_attn_fwd_fp8_workspace_size.restype = sz
    lib.fa_attn_fwd_fp8.argtypes = [pp, vp, vp, vp, f, f, f, vp, vp, vp, sz, vp]
    lib.fa_attn_fwd_fp8.restype = i
    lib.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    lib.fa_bwd_noalloc.restype = i
    lib.fa_selftest_wait_timeout.argtypes = [vp]
    lib.fa_selftest_wait_timeout.restype = i
    lib.fa_selftest_exp2.argtypes = [vp, vp, i, vp]
    lib.fa_selftest_exp2.restype = i
    lib.fa_last_device_status.argtypes = [vp]
    lib.fa_last_device_status.restype = i
    lib.fa_device_status.argtypes = [vp]
    lib.fa_device_status.restype = i
    lib.fa_bwd_set_phase_events.argtypes = [vp]
    lib.fa_bwd_set_phase_events.restype = None
    lib.fa_status_str.argtypes = [i]
    lib.fa_status_str.restype = ctypes.c_char_p
    _LIB = lib
    return lib


def status_str(status: int) -> str:
    return library().fa_status_str(int(status)).decode()


fa_status_str = status_str


def _stream_handle(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _check(fn: str, status: int) -> None:
    if status != FA_OK:
        raise FAError(fn, status)


def _shape(q: torch.Tensor) -> tuple[int, int, int, int]:
    if q.dim() != 4:
        raise ValueError("expected a (B, H, N, d) tensor")
    return tuple(int(x) for x in q.shape)  # type: ignore[return-value]


def _same(*ts: torch.Tensor, dtype: torch.dtype, shape) -> None:
    for t in ts:
        if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"expected contiguous CUDA {dtype} tensors of shape {tuple(shape)}")


def _scale(scale, d: int) -> float:
    return float(1.0 / math.sqrt(d) if scale is None else scale)


def fa_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False, scale: float | None = None,
           o: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None):
    """Attention forward on bf16 (B, H, N, d) CUDA tensors (C ``fa_fwd``).  Returns (o, lse).

    The residual a training forward can hand to the backward is written by ``fa_fwd_gqa``,
    ``fa_fwd_ws`` and ``fa_attn_fwd`` (``save_residual=True``)."""
    B, H, N, d = _shape(q)
    _same(q, k, v, dtype=torch.bfloat16, shape=(B, H, N, d))
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _same(o, dtype=torch.bfloat16, shape=(B, H, N, d))
    _same(lse, dtype=torch.float32, shape=(B, H, N))
    st = library().fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N, d,
                          _scale(scale, d), int(bool(causal)), _stream_handle(stream))
    _check("fa_fwd", st)
    return o, lse


def _gqa_heads(q: torch.Tensor, k: torch.Tensor) -> int:
    if k.dim() != 4 or k.shape[0] != q.shape[0] or k.shape[2:] != q.shape[2:]:
        raise ValueError("k, v must be (B, H_kv, N, d) with q's B, N and d")
    h_kv = int(k.shape[1])
    if h_kv < 1 or q.shape[1] % h_kv:
        raise ValueError("the query head count must be a multiple of the key/value head count")
    return h_kv


def fa_fwd_gqa(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
               scale: float | None = None, o: torch.Tensor | None = None, lse: torch.Tensor | None = None,
               o_resid: torch.Tensor | None = None, save_residual: bool = False, stream=None):
    """Grouped-query / multi-query forward: q (B, H, N, d), k and v (B, H_kv, N, d) bf16.

    Query head h reads key/value head h // (H // H_kv).  Returns like ``fa_fwd``."""
    B, H, N, d = _shape(q)
    H_kv = _gqa_heads(q, k)
    _same(q, dtype=torch.bfloat16, shape=(B, H, N, d))
    _same(k, v, dtype=torch.bfloat16, shape=(B, H_kv, N, d))
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if o_resid is None and save_residual:
        o_resid = torch.empty_like(q)
    _same(o, dtype=torch.bfloat16, shape=(B, H, N, d))
    if o_resid is not None:
        _same(o_resid, dtype=torch.bfloat16, shape=(B, H, N, d))
    st = library().fa_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                              None if o_resid is None else o_resid.data_ptr(), B, H, H_kv, N, d, _scale(scale, d),
                              int(bool(causal)), _stream_handle(stream))
    _check("fa_fwd_gqa", st)
    return (o, lse) if o_resid is None else (o, lse, o_resid)


def fa_fwd_workspace_size(B: int, H_kv: int, N: int, d: int) -> int:
    return int(library().fa_fwd_workspace_size(B, H_kv, N, d))


def fa_fwd_ws(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
              scale: float | None = None, o: torch.Tensor | None = None, lse: torch.Tensor | None = None,
              o_resid: torch.Tensor | None = None, save_residual: bool = False, workspace=None, stream=None):
    """Forward with a workspace (V converted to fp16 in one pass before the kernel); k, v may
    have fewer heads than q (grouped-query).  Returns like ``fa_fwd``."""
    B, H, N, d = _shape(q)
    H_kv = _gqa_heads(q, k)
    _same(q, dtype=torch.bfloat16, shape=(B, H, N, d))
    _same(k, v, dtype=torch.bfloat16, shape=(B, H_kv, N, d))
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if o_resid is None and save_residual:
        o_resid = torch.empty_like(q)
    _same(o, dtype=torch.bfloat16, shape=(B, H, N, d))
    if o_resid is not None:
        _same(o_resid, dtype=torch.bfloat16, shape=(B, H, N, d))
    if workspace is None:
        workspace = torch.empty(max(fa_fwd_workspace_size(B, H_kv, N, d), 1), dtype=torch.uint8, device=q.device)
    st = library().fa_fwd_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                             None if o_resid is None else o_resid.data_ptr(), B, H, H_kv, N, d, _scale(scale, d),
                             int(bool(causal)), workspace.data_ptr(), workspace.numel(), _stream_handle(stream))
    _check("fa_fwd_ws", st)
    return (o, lse) if o_resid is None else (o, lse, o_resid)


def fa_fwd_f32(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
               scale: float | None = None, stream=None):
    """fp32 forward (no input rounding). Returns (o, lse)."""
    B, H, N, d = _shape(q)
    _same(q, k, v, dtype=torch.float32, shape=(B, H, N, d))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    st = library().fa_fwd_f32(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N, d,
                              _scale(scale, d), int(bool(causal)), _stream_handle(stream))
    _check("fa_fwd_f32", st)
    return o, lse


def fa_bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(library().fa_bwd_workspace_size(B, H, N, d))


def fa_bwd(q, k, v, o, do, lse, causal: bool = False, scale: float | None = None, workspace=None,
           dq=None, dk=None, dv=None, stream=None):
    """dQ, dK, dV (fp32) of sum(O * dO) (C ``fa_bwd``; rowsum(dO * O) from the bf16 O --
    ``fa_bwd_gqa`` / ``fa_attn_bwd`` take the forward's residual).  Returns (dq, dk, dv)."""
    B, H, N, d = _shape(q)
    _same(q, k, v, o, do, dtype=torch.bfloat16, shape=(B, H, N, d))
    _same(lse, dtype=torch.float32, shape=(B, H, N))
    if dq is None:
        dq = torch.empty((B, H, N, d), dtype=torch.float32, device=q.device)
    if dk is None:
        dk = torch.empty_like(dq)
    if dv is None:
        dv = torch.empty_like(dq)
    _same(dq, dk, dv, dtype=torch.float32, shape=(B, H, N, d))
    ws_bytes = fa_bwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    if workspace.numel() < ws_bytes:  # the C call trusts the size (its signature carries none)
        raise ValueError(f"workspace of {workspace.numel()} bytes, fa_bwd needs {ws_bytes}")
    st = library().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                          dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, _scale(scale, d),
                          int(bool(causal)), workspace.data_ptr(), _stream_handle(stream))
    _check("fa_bwd", st)
    return dq, dk, dv


def fa_bwd_gqa_workspace_size(B: int, H: int, H_kv: int, N: int, d: int) -> int:
    return int(library().fa_bwd_gqa_workspace_size(B, H, H_kv, N, d))


def fa_bwd_gqa(q, k, v, o, do, lse, causal: bool = False, scale: float | None = None, workspace=None,
               dq=None, dk=None, dv=None, o_resid=None, stream=None):
    """Grouped-query backward: dq (B, H, N, d); dk, dv (B, H_kv, N, d), summed over each group."""
    B, H, N, d = _shape(q)
    H_kv = _gqa_heads(q, k)
    _same(q, o, do, dtype=torch.bfloat16, shape=(B, H, N, d))
    _same(k, v, dtype=torch.bfloat16, shape=(B, H_kv, N, d))
    _same(lse, dtype=torch.float32, shape=(B, H, N))
    if o_resid is not None:
        _same(o_resid, dtype=torch.bfloat16, shape=(B, H, N, d))
    if dq is None:
        dq = torch.empty((B, H, N, d), dtype=torch.float32, device=q.device)
    if dk is None:
        dk = torch.empty((B, H_kv, N, d), dtype=torch.float32, device=q.device)
    if dv is None:
        dv = torch.empty_like(dk)
    _same(dq, dtype=torch.float32, shape=(B, H, N, d))
    _same(dk, dv, dtype=torch.float32, shape=(B, H_kv, N, d))
    ws_bytes = fa_bwd_gqa_workspace_size(B, H, H_kv, N, d)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    st = library().fa_bwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              None if o_resid is None else o_resid.data_ptr(), do.data_ptr(), lse.data_ptr(),
                              dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, H_kv, N, d, _scale(scale, d),
                              int(bool(causal)), workspace.data_ptr(), workspace.numel(), _stream_handle(stream))
    _check("fa_bwd_gqa", st)
    return dq, dk, dv


def fa_bwd_ws_workspace_size(B: int, H: int, H_kv: int, N: int, d: int) -> int:
    return int(library().fa_bwd_ws_workspace_size(B, H, H_kv, N, d))


def fa_bwd_ws(q, k, v, o, do, lse, fwd_workspace, causal: bool = False, scale: float | None = None,
              workspace=None, dq=None, dk=None, dv=None, o_resid=None, stream=None):
    """``fa_bwd_gqa`` that takes the fp16 V copy from ``fwd_workspace``, the workspace of the
    ``fa_fwd_ws`` call that produced o (and lse, o_resid) from this v.  Returns (dq, dk, dv)."""
    B, H, N, d = _shape(q)
    H_kv = _gqa_heads(q, k)
    _same(q, o, do, dtype=torch.bfloat16, shape=(B, H, N, d))
    _same(k, v, dtype=torch.bfloat16, shape=(B, H_kv, N, d))
    _same(lse, dtype=torch.float32, shape=(B, H, N))
    if o_resid is not None:
        _same(o_resid, dtype=torch.bfloat16, shape=(B, H, N, d))
    if fwd_workspace is None or fwd_workspace.device != q.device:
        raise ValueError("fa_bwd_ws needs the forward's workspace on the inputs' device")
    if dq is None:
        dq = torch.empty((B, H, N, d), dtype=torch.float32, device=q.device)
    if dk is None:
        dk = torch.empty((B, H_kv, N, d), dtype=torch.float32, device=q.device)
    if dv is None:
        dv = torch.empty_like(dk)
    _same(dq, dtype=torch.float32, shape=(B, H, N, d))
    _same(dk, dv, dtype=torch.float32, shape=(B, H_kv, N, d))
    if workspace is None:
        workspace = torch.empty(max(fa_bwd_ws_workspace_size(B, H, H_kv, N, d), 1), dtype=torch.uint8,
                                device=q.device)
    st = library().fa_bwd_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                             None if o_resid is None else o_resid.data_ptr(), do.data_ptr(), lse.data_ptr(),
                             dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, H_kv, N, d, _scale(scale, d),
                             int(bool(causal)), fwd_workspace.data_ptr(), fwd_workspace.numel(),
                             workspace.data_ptr(), workspace.numel(), _stream_handle(stream))
    _check("fa_bwd_ws", st)
    return dq, dk, dv


def _problem(q, k, causal, scale, window) -> FaAttnProblem:
    B, H, N, d = _shape(q)
    H_kv = _gqa_heads(q, k)
    wl, wr = window
    return FaAttnProblem(B, H, H_kv, N, d, _scale(scale, d), int(bool(causal)), int(wl), int(wr))


def fa_attn_fwd_workspace_size(problem: FaAttnProblem) -> int:
    return int(library().fa_attn_fwd_workspace_size(ctypes.byref(problem)))


def fa_attn_bwd_workspace_size(problem: FaAttnProblem) -> int:
    return int(library().fa_attn_bwd_workspace_size(ctypes.byref(problem)))


def fa_attn_fwd(q, k, v, causal: bool = False, scale: float | None = None, window=(-1, -1), o=None, lse=None,
                o_resid=None, save_residual: bool = False, workspace=None, stream=None):
    """Forward with every option: grouped K/V heads (k, v (B, H_kv, N, d)) and a sliding
    window (left, right) (-1 = unbounded).  Returns like ``fa_fwd``."""
    pr = _problem(q, k, causal, scale, window)
    B, H, N, d = _shape(q)
    _same(q, dtype=torch.bfloat16, shape=(B, H, N, d))
    _same(k, v, dtype=torch.bfloat16, shape=(B, pr.H_kv, N, d))
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if o_resid is None and save_residual:
        o_resid = torch.empty_like(q)
    _same(o, dtype=torch.bfloat16, shape=(B, H, N, d))
    if o_resid is not None:
        _same(o_resid, dtype=torch.bfloat16, shape=(B, H, N, d))
    if workspace is None:
        workspace = torch.empty(max(fa_attn_fwd_workspace_size(pr), 1), dtype=torch.uint8, device=q.device)
    st = library().fa_attn_fwd(ctypes.byref(pr), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                               lse.data_ptr(), None if o_resid is None else o_resid.data_ptr(), workspace.data_ptr(),
                               workspace.numel(), _stream_handle(stream))
    _check("fa_attn_fwd", st)
    return (o, lse) if o_resid is None else (o, lse, o_resid)


def fa_attn_fwd_fp8_workspace_size(problem: FaAttnProblem) -> int:
    return int(library().fa_attn_fwd_fp8_workspace_size(ctypes.byref(problem)))


def fa_attn_fwd_fp8(q, k, v, q_descale: float, k_descale: float, v_descale: float, causal: bool = False,
                    scale: float | None = None, window=(-1, -1), o=None, lse=None, workspace=None, stream=None):
    """8-bit forward: q (B, H, N, d), k and v (B, H_kv, N, d) ``torch.float8_e4m3fn`` CUDA
    tensors holding Q / q_descale etc. (per-tensor descales, d = 128 or 64).  Computes the
    attention of the dequantized inputs; returns (o bf16, lse fp32)."""
    pr = _problem(q, k, causal, scale, window)
    B, H, N, d = _shape(q)
    _same(q, dtype=torch.float8_e4m3fn, shape=(B, H, N, d))
    _same(k, v, dtype=torch.float8_e4m3fn, shape=(B, pr.H_kv, N, d))
    if o is None:
        o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _same(o, dtype=torch.bfloat16, shape=(B, H, N, d))
    _same(lse, dtype=torch.float32, shape=(B, H, N))
    if workspace is None:
        workspace = torch.empty(max(fa_attn_fwd_fp8_workspace_size(pr), 1), dtype=torch.uint8, device=q.device)
    st = library().fa_attn_fwd_fp8(ctypes.byref(pr), q.data_ptr(), k.data_ptr(), v.data_ptr(), float(q_descale),
                                   float(k_descale), float(v_descale), o.data_ptr(), lse.data_ptr(),
                                   workspace.data_ptr(), workspace.numel(), _stream_handle(stream))
    _check("fa_attn_fwd_fp8", st)
    return o, lse


def fa_attn_bwd(q, k, v, o, do, lse, causal: bool = False, scale: float | None = None, window=(-1, -1),
                workspace=None, dq=None, dk=None, dv=None, o_resid=None, stream=None):
    """Backward with every option (the same problem as the forward).  Returns (dq, dk, dv)."""
    pr = _problem(q, k, causal, scale, window)
    B, H, N, d = _shape(q)
    _same(q, o, do, dtype=torch.bfloat16, shape=(B, H, N, d))
    _same(k, v, dtype=torch.bfloat16, shape=(B, pr.H_kv, N, d))
    _same(lse, dtype=torch.float32, shape=(B, H, N))
    if o_resid is not None:
        _same(o_resid, dtype=torch.bfloat16, shape=(B, H, N, d))
    if dq is None:
        dq = torch.empty((B, H, N, d), dtype=torch.float32, device=q.device)
    if dk is None:
        dk = torch.empty((B, pr.H_kv, N, d), dtype=torch.float32, device=q.device)
    if dv is None:
        dv = torch.empty_like(dk)
    _same(dq, dtype=torch.float32, shape=(B, H, N, d))
    _same(dk, dv, dtype=torch.float32, shape=(B, pr.H_kv, N, d))
    if workspace is None:
        workspace = torch.empty(max(fa_attn_bwd_workspace_size(pr), 1), dtype=torch.uint8, device=q.device)
    st = library().fa_attn_bwd(ctypes.byref(pr), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                               None if o_resid is None else o_resid.data_ptr(), do.data_ptr(), lse.data_ptr(),
                               dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(), workspace.numel(),
                               _stream_handle(stream))
    _check("fa_attn_bwd", st)
    return dq, dk, dv


def fa_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, causal: bool = False, scale: float | None = None,
                   o_resid=None, stream=None):
    """The backward pass without a workspace, for callers that cannot allocate device memory
    when they run it: the C entry point uses a scratch array built into the library (64 MiB
    per GPU, shared by all calls on that GPU, so overlapping calls race).  The caller passes
    every input and the fp32 outputs dq, dk, dv; nothing is allocated here either."""
    B, H, N, d = _shape(q)
    _same(q, k, v, o, do, dtype=torch.bfloat16, shape=(B, H, N, d))
    _same(lse, dtype=torch.float32, shape=(B, H, N))
    _same(dq, dk, dv, dtype=torch.float32, shape=(B, H, N, d))
    if o_resid is not None:
        _same(o_resid, dtype=torch.bfloat16, shape=(B, H, N, d))
    st = library().fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  None if o_resid is None else o_resid.data_ptr(), do.data_ptr(), lse.data_ptr(),
                                  dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, _scale(scale, d),
                                  int(bool(causal)), _stream_handle(stream))
    _check("fa_bwd_noalloc", st)
    return dq, dk, dv


def fa_selftest_wait_timeout(stream=None) -> None:
    """Enqueue the bounded-wait self-test (a wait that must give up after ~2 s and report
    FA_ERR_TIMEOUT through ``fa_device_status``)."""
    _check("fa_selftest_wait_timeout", library().fa_selftest_wait_timeout(_stream_handle(stream)))


def fa_selftest_exp2(x: torch.Tensor, stream=None) -> torch.Tensor:
    """The FMA-pipe exponential of the softmax kernels applied to a 1-D fp32 CUDA tensor."""
    if x.dtype != torch.float32 or x.dim() != 1 or not x.is_contiguous() or not x.is_cuda:
        raise ValueError("expected a contiguous 1-D fp32 CUDA tensor")
    y = torch.empty_like(x)
    _check("fa_selftest_exp2", library().fa_selftest_exp2(x.data_ptr(), y.data_ptr(), x.numel(),
                                                          _stream_handle(stream)))
    return y


def fa_last_device_status(stream=None) -> int:
    """Synchronise and return (and clear) the device status code: FA_OK, FA_ERR_TIMEOUT,
    FA_ERR_RANGE or FA_ERR_CUDA."""
    return int(library().fa_last_device_status(_stream_handle(stream)))


def fa_device_status(stream=None) -> int:
    """``fa_last_device_status`` under its earlier name."""
    return int(library().fa_device_status(_stream_handle(stream)))


_PHASE_EVENTS = None  # keeps the ctypes array alive while the hook is set


def fa_bwd_set_phase_events(events=None) -> None:
    """Profiling hook: record ``events[0]`` after the preprocess and ``events[1]`` after the
    dK/dV kernel in every later ``fa_bwd`` of this thread (``torch.cuda.Event`` objects);
    ``None`` turns it off."""
    global _PHASE_EVENTS
    if events is None:
        _PHASE_EVENTS = None
        library().fa_bwd_set_phase_events(None)
        return
    for ev in events[:2]:
        if not ev.cuda_event:  # torch creates the CUDA event lazily, on its first record
            ev.record()
    arr = (ctypes.c_void_p * 2)(events[0].cuda_event, events[1].cuda_event)
    _PHASE_EVENTS = arr
    library().fa_bwd_set_phase_events(ctypes.cast(arr, ctypes.c_void_p))
