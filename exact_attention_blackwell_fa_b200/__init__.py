"""Exact scaled-dot-product attention (forward and backward) for B200 / sm_100a.

Thin Python binding over the C ABI in include/fa.h (libfa.so).  PyTorch supplies
device memory and the current stream; every step of the computation runs in the
library's CUDA kernels.  The functions carry the C names:

    fa_fwd(q, k, v, causal=False, scale=None) -> (o, lse)
    fa_fwd_splitkv(q, k, v, causal=False, scale=None, num_splits=0) -> (o, lse)
    fa_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                  seqused_k=None, causal=False, scale=None) -> (o, lse)
    fa_bwd(q, k, v, o, lse, dout, causal=False, scale=None) -> (dq, dk, dv)
    fa_bwd_varlen(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                  max_seqlen_k, seqused_k=None, causal=False, scale=None) -> (dq, dk, dv)
    fa_bwd_workspace_size(B, Sq, Hq, d) -> int
    fa_bwd_noalloc(q, k, v, o, lse, dout, causal=False, scale=None) -> (dq, dk, dv)
    fa_status_string(code) -> str
    fa_last_device_status() -> (code, detail)
    fa_clear_device_status()
    fa_set_unit_schedule(mode)        # FA_SCHED_STATIC (0, default) or FA_SCHED_CLC (1)
    fa_debug_inject(mode)
    fa_debug_exp2(x, mode=0) -> y

Tensors are CUDA, contiguous, [batch, seq, heads, head_dim], bf16 or fp16; LSE is
float32 [batch, Hq, Sq].  A non-OK status raises FAError; nothing falls back.
"""
from __future__ import annotations

import ctypes
import math

import torch

from . import _lib

__all__ = [
    "FAError", "fa_fwd", "fa_fwd_splitkv", "fa_fwd_varlen", "fa_bwd", "fa_bwd_varlen", "fa_bwd_noalloc", "fa_bwd_workspace_size", "fa_status_string",
    "fa_last_device_status", "fa_clear_device_status", "fa_set_unit_schedule", "fa_debug_inject", "fa_debug_exp2",
    "FA_SCHED_STATIC", "FA_SCHED_CLC",
]

FA_SCHED_STATIC, FA_SCHED_CLC = 0, 1


class FAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {fa_status_string(code)}")


def fa_status_string(code: int) -> str:
    return _lib.load().fa_status_string(int(code)).decode()


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return _lib.FA_BF16
    if t.dtype == torch.float16:
        return _lib.FA_FP16
    raise TypeError(f"fa: inputs must be bf16 or fp16, got {t.dtype}")


def _check(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"fa: {name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"fa: {name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"fa: {name} has dtype {t.dtype}, expected {dtype}")


def _raise(code: int, where: str):
    if code != _lib.FA_OK:
        raise FAError(code, where)


def fa_fwd(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
           stream=None):
    """Forward. q [B,Sq,Hq,d], k/v [B,Sk,Hkv,d] -> (o [B,Sq,Hq,d], lse [B,Hq,Sq] fp32)."""
    _check(q, "q")
    _check(k, "k", q.dtype)
    _check(v, "v", q.dtype)
    B, Sq, Hq, d = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if k.shape != v.shape or k.shape[0] != B or k.shape[3] != d:
        raise ValueError("fa: k and v must be [B, Sk, Hkv, d] matching q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, Sq, dtype=torch.float32, device=q.device)
    _check(out, "out", q.dtype)
    _check(lse, "lse", torch.float32)
    code = _lib.load().fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                              lse.data_ptr(), B, Sq, Sk, Hq, Hkv, d, int(bool(causal)),
                              float(scale), _dtype_code(q), _stream_ptr(stream))
    _raise(code, "fa_fwd")
    return out, lse


def fa_fwd_splitkv(q, k, v, causal: bool = False, scale: float | None = None, num_splits: int = 0,
                   out=None, lse=None, workspace=None, stream=None):
    """Split-KV forward (decode-shaped calls): same layouts and result as fa_fwd.
    num_splits <= 0 lets the library choose."""
    _check(q, "q")
    _check(k, "k", q.dtype)
    _check(v, "v", q.dtype)
    B, Sq, Hq, d = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if k.shape != v.shape or k.shape[0] != B or k.shape[3] != d:
        raise ValueError("fa: k and v must be [B, Sk, Hkv, d] matching q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty(B, Hq, Sq, dtype=torch.float32, device=q.device)
    lib = _lib.load()
    if workspace is None:
        need = int(lib.fa_fwd_splitkv_workspace_size(B, Sq, Sk, Hq, Hkv, d, int(num_splits)))
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    code = lib.fa_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Sq,
                              Sk, Hq, Hkv, d, int(bool(causal)), float(scale), _dtype_code(q), int(num_splits),
                              workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    _raise(code, "fa_fwd_splitkv")
    return out, lse


def fa_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                  seqused_k=None, causal: bool = False, scale: float | None = None, out=None, lse=None,
                  stream=None):
    """Forward over packed variable-length sequences.  q [total_q,Hq,d], k/v
    [total_k,Hkv,d], cu_seqlens_* int32 CUDA [B+1], seqused_k int32 CUDA [B] or None
    -> (o [total_q,Hq,d], lse [Hq,total_q] fp32)."""
    _check(q, "q")
    _check(k, "k", q.dtype)
    _check(v, "v", q.dtype)
    total_q, Hq, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    if k.shape != v.shape or k.shape[2] != d:
        raise ValueError("fa: k and v must be [total_k, Hkv, d] matching q")
    for name, t in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)) + (
            (("seqused_k", seqused_k),) if seqused_k is not None else ()):
        if t.device.type != "cuda" or t.dtype != torch.int32 or not t.is_contiguous():
            raise ValueError(f"fa: {name} must be a contiguous CUDA int32 tensor")
    B = cu_seqlens_q.numel() - 1
    if B < 1 or cu_seqlens_k.numel() != B + 1 or (seqused_k is not None and seqused_k.numel() != B):
        raise ValueError("fa: cu_seqlens_q / cu_seqlens_k need B+1 entries, seqused_k B")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(Hq, total_q, dtype=torch.float32, device=q.device)
    _check(out, "out", q.dtype)
    _check(lse, "lse", torch.float32)
    code = _lib.load().fa_fwd_varlen(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), cu_seqlens_q.data_ptr(),
        cu_seqlens_k.data_ptr(), seqused_k.data_ptr() if seqused_k is not None else None, B,
        int(max_seqlen_q), int(max_seqlen_k), total_q, total_k, Hq, Hkv, d, int(bool(causal)),
        float(scale), _dtype_code(q), _stream_ptr(stream))
    _raise(code, "fa_fwd_varlen")
    return out, lse


def fa_bwd_workspace_size(B: int, Sq: int, Hq: int, d: int) -> int:
    return int(_lib.load().fa_bwd_workspace_size(B, Sq, Hq, d))


def fa_bwd(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None,
           dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Backward. Returns (dq, dk, dv) in the input dtype."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check(t, name, q.dtype)
    _check(lse, "lse", torch.float32)
    B, Sq, Hq, d = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ws_bytes = fa_bwd_workspace_size(B, Sq, Hq, d)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    code = _lib.load().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                              dv.data_ptr(), B, Sq, Sk, Hq, Hkv, d, int(bool(causal)),
                              float(scale), _dtype_code(q), workspace.data_ptr(),
                              workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    _raise(code, "fa_bwd")
    return dq, dk, dv


def fa_bwd_varlen(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                  max_seqlen_k: int, seqused_k=None, causal: bool = False, scale: float | None = None,
                  dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Backward over packed variable-length sequences (layouts as fa_fwd_varlen)
    -> (dq [total_q,Hq,d], dk, dv [total_k,Hkv,d])."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _check(t, n, q.dtype)
    _check(lse, "lse", torch.float32)
    total_q, Hq, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    for name, t in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)) + (
            (("seqused_k", seqused_k),) if seqused_k is not None else ()):
        if t.device.type != "cuda" or t.dtype != torch.int32 or not t.is_contiguous():
            raise ValueError(f"fa: {name} must be a contiguous CUDA int32 tensor")
    B = cu_seqlens_q.numel() - 1
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = fa_bwd_workspace_size(B, int(max_seqlen_q), Hq, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    code = _lib.load().fa_bwd_varlen(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), dout.data_ptr(),
        dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(),
        seqused_k.data_ptr() if seqused_k is not None else None, B, int(max_seqlen_q), int(max_seqlen_k),
        total_q, total_k, Hq, Hkv, d, int(bool(causal)), float(scale), _dtype_code(q), workspace.data_ptr(),
        workspace.numel(), _stream_ptr(stream))
    _raise(code, "fa_bwd_varlen")
    return dq, dk, dv


def fa_bwd_noalloc(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None,
                   dq=None, dk=None, dv=None, stream=None):
    """Backward without a workspace: the library keeps the scratch in a fixed device
    array (for callers that cannot allocate device memory).  Calls that overlap on
    the GPU race on that array.  Output tensors may be passed in to avoid allocating
    them here too.  Returns (dq, dk, dv)."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check(t, name, q.dtype)
    _check(lse, "lse", torch.float32)
    B, Sq, Hq, d = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    code = _lib.load().fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                      lse.data_ptr(), dout.data_ptr(), dq.data_ptr(),
                                      dk.data_ptr(), dv.data_ptr(), B, Sq, Sk, Hq, Hkv, d,
                                      int(bool(causal)), float(scale), _dtype_code(q),
                                      _stream_ptr(stream))
    _raise(code, "fa_bwd_noalloc")
    return dq, dk, dv


def fa_last_device_status(stream=None):
    """(code, detail) of the device status word; synchronises the stream."""
    detail = ctypes.c_uint32(0)
    code = _lib.load().fa_last_device_status(_stream_ptr(stream), ctypes.byref(detail))
    return int(code), int(detail.value)


def fa_clear_device_status(stream=None):
    _raise(_lib.load().fa_clear_device_status(_stream_ptr(stream)), "fa_clear_device_status")


def fa_set_unit_schedule(mode: int):
    """Forward unit order: FA_SCHED_STATIC (persistent grid, fixed stride; default) or
    FA_SCHED_CLC (one CTA per unit, running CTAs cancel pending ones to take their
    units).  Process-wide."""
    _raise(_lib.load().fa_set_unit_schedule(int(mode)), "fa_set_unit_schedule")


def fa_debug_inject(mode: int):
    _raise(_lib.load().fa_debug_inject(int(mode)), "fa_debug_inject")


def fa_debug_exp2(x, mode: int = 0, stream=None):
    """The kernels' exp2 on a CUDA fp32 tensor: mode 0 the FMA-pipe cubic, 1 the SFU
    instruction.  Returns a new tensor (enqueued on the stream)."""
    if x.device.type != "cuda" or x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA float32 tensor")
    y = torch.empty_like(x)
    _raise(_lib.load().fa_debug_exp2(x.data_ptr(), y.data_ptr(), x.numel(), int(mode), _stream_ptr(stream)),
           "fa_debug_exp2")
    return y
