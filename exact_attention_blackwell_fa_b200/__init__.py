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
    fa_set_unit_schedule(mode)        # FA_SCHED_STATIC (0), FA_SCHED_CLC (1), FA_SCHED_AUTO (2, default)
    fa_set_exp2_emulation(pairs_of_4) # forward exp2 split: -1 default, 0..3 of 4 on the FMA pipe
    fa_set_wait_timeout_ms(ms)        # limit of a kernel's pipeline waits (default 1000)
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
    "fa_last_device_status", "fa_clear_device_status", "fa_set_unit_schedule", "fa_set_exp2_emulation", "fa_set_wait_timeout_ms", "fa_debug_inject", "fa_debug_exp2",
    "FA_SCHED_STATIC", "FA_SCHED_CLC", "FA_SCHED_AUTO",
]

FA_SCHED_STATIC, FA_SCHED_CLC, FA_SCHED_AUTO = 0, 1, 2


class FAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {fa_status_string(code)}")


def fa_status_string(code: int) -> str:
    return _lib.load().fa_status_string(int(code)).decode()


def _stream_ptr(stream) -> int:
    """The stream handle to launch on: the given one, else the current device's current
    stream (the wrappers make q's device current first)."""
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


def _same_device(ref: torch.Tensor, **tensors):
    """Every tensor must sit on ref's device: the library launches on the current
    device, which the wrappers set to ref's."""
    for name, t in tensors.items():
        if t is not None and t.device != ref.device:
            raise ValueError(f"fa: {name} is on {t.device}, expected {ref.device}")


def _shape(t: torch.Tensor, name: str, shape):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"fa: {name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _check_kv(q, k, v, packed: bool):
    if packed:
        if q.dim() != 3 or k.dim() != 3 or k.shape != v.shape or k.shape[2] != q.shape[2]:
            raise ValueError("fa: q must be [total_q, Hq, d] and k, v [total_k, Hkv, d] with the same d")
    elif q.dim() != 4 or k.dim() != 4 or k.shape != v.shape or k.shape[0] != q.shape[0] or \
            k.shape[3] != q.shape[3]:
        raise ValueError("fa: q must be [B, Sq, Hq, d] and k, v [B, Sk, Hkv, d] matching q")


def _workspace(ws, ref: torch.Tensor, need: int, name: str = "workspace"):
    if ws is None:
        return torch.empty(max(need, 256), dtype=torch.uint8, device=ref.device)
    _check(ws, name)
    _same_device(ref, **{name: ws})
    if ws.numel() * ws.element_size() < need:
        raise ValueError(f"fa: {name} holds {ws.numel() * ws.element_size()} bytes, needs {need}")
    return ws


def _raise(code: int, where: str):
    if code != _lib.FA_OK:
        raise FAError(code, where)


def fa_fwd(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
           stream=None):
    """Forward. q [B,Sq,Hq,d], k/v [B,Sk,Hkv,d] -> (o [B,Sq,Hq,d], lse [B,Hq,Sq] fp32)."""
    _check(q, "q")
    _check(k, "k", q.dtype)
    _check(v, "v", q.dtype)
    _check_kv(q, k, v, packed=False)
    B, Sq, Hq, d = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, Sq, dtype=torch.float32, device=q.device)
    _check(out, "out", q.dtype)
    _check(lse, "lse", torch.float32)
    _shape(out, "out", q.shape)
    _shape(lse, "lse", (B, Hq, Sq))
    _same_device(q, k=k, v=v, out=out, lse=lse)
    with torch.cuda.device(q.device):
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
    _check_kv(q, k, v, packed=False)
    B, Sq, Hq, d = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty(B, Hq, Sq, dtype=torch.float32, device=q.device)
    _check(out, "out", q.dtype)
    _check(lse, "lse", torch.float32)
    _shape(out, "out", q.shape)
    _shape(lse, "lse", (B, Hq, Sq))
    _same_device(q, k=k, v=v, out=out, lse=lse)
    lib = _lib.load()
    with torch.cuda.device(q.device):
        need = int(lib.fa_fwd_splitkv_workspace_size(B, Sq, Sk, Hq, Hkv, d, int(num_splits)))
        workspace = _workspace(workspace, q, need)
        code = lib.fa_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B,
                                  Sq, Sk, Hq, Hkv, d, int(bool(causal)), float(scale), _dtype_code(q),
                                  int(num_splits), workspace.data_ptr(),
                                  workspace.numel() * workspace.element_size(), _stream_ptr(stream))
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
    _check_kv(q, k, v, packed=True)
    total_q, Hq, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    B = _check_seqlens(q, cu_seqlens_q, cu_seqlens_k, seqused_k)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(Hq, total_q, dtype=torch.float32, device=q.device)
    _check(out, "out", q.dtype)
    _check(lse, "lse", torch.float32)
    _shape(out, "out", q.shape)
    _shape(lse, "lse", (Hq, total_q))
    _same_device(q, k=k, v=v, out=out, lse=lse)
    with torch.cuda.device(q.device):
        code = _lib.load().fa_fwd_varlen(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), cu_seqlens_q.data_ptr(),
            cu_seqlens_k.data_ptr(), seqused_k.data_ptr() if seqused_k is not None else None, B,
            int(max_seqlen_q), int(max_seqlen_k), total_q, total_k, Hq, Hkv, d, int(bool(causal)),
            float(scale), _dtype_code(q), _stream_ptr(stream))
    _raise(code, "fa_fwd_varlen")
    return out, lse


def _check_seqlens(q, cu_seqlens_q, cu_seqlens_k, seqused_k) -> int:
    """Validates the sequence-boundary arrays of a packed batch; returns B."""
    for name, t in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)) + (
            (("seqused_k", seqused_k),) if seqused_k is not None else ()):
        if not isinstance(t, torch.Tensor) or t.device != q.device or t.dtype != torch.int32 or \
                not t.is_contiguous():
            raise ValueError(f"fa: {name} must be a contiguous int32 tensor on {q.device}")
    B = cu_seqlens_q.numel() - 1
    if B < 1 or cu_seqlens_k.numel() != B + 1 or (seqused_k is not None and seqused_k.numel() != B):
        raise ValueError("fa: cu_seqlens_q / cu_seqlens_k need B+1 entries, seqused_k B")
    return B


def _check_bwd_tensors(q, k, v, o, lse, dout, dq, dk, dv, lse_shape):
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout), ("dq", dq), ("dk", dk),
                    ("dv", dv)):
        _check(t, name, q.dtype)
    _check(lse, "lse", torch.float32)
    for name, t in (("o", o), ("dout", dout), ("dq", dq)):
        _shape(t, name, q.shape)
    _shape(dk, "dk", k.shape)
    _shape(dv, "dv", k.shape)
    _shape(lse, "lse", lse_shape)
    _same_device(q, k=k, v=v, o=o, lse=lse, dout=dout, dq=dq, dk=dk, dv=dv)


def fa_bwd_workspace_size(B: int, Sq: int, Hq: int, d: int) -> int:
    return int(_lib.load().fa_bwd_workspace_size(B, Sq, Hq, d))


def fa_bwd(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None,
           dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Backward. Returns (dq, dk, dv) in the input dtype."""
    _check(q, "q")
    _check_kv(q, k, v, packed=False)
    B, Sq, Hq, d = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_bwd_tensors(q, k, v, o, lse, dout, dq, dk, dv, (B, Hq, Sq))
    with torch.cuda.device(q.device):
        workspace = _workspace(workspace, q, fa_bwd_workspace_size(B, Sq, Hq, d))
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
    _check(q, "q")
    _check_kv(q, k, v, packed=True)
    total_q, Hq, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    B = _check_seqlens(q, cu_seqlens_q, cu_seqlens_k, seqused_k)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_bwd_tensors(q, k, v, o, lse, dout, dq, dk, dv, (Hq, total_q))
    with torch.cuda.device(q.device):
        workspace = _workspace(workspace, q, fa_bwd_workspace_size(B, int(max_seqlen_q), Hq, d))
        code = _lib.load().fa_bwd_varlen(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), dout.data_ptr(),
            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(),
            seqused_k.data_ptr() if seqused_k is not None else None, B, int(max_seqlen_q), int(max_seqlen_k),
            total_q, total_k, Hq, Hkv, d, int(bool(causal)), float(scale), _dtype_code(q), workspace.data_ptr(),
            workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    _raise(code, "fa_bwd_varlen")
    return dq, dk, dv


def fa_bwd_noalloc(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None,
                   dq=None, dk=None, dv=None, stream=None):
    """Backward without a workspace: the library keeps the scratch in a fixed device
    array (for callers that cannot allocate device memory).  Calls that overlap on
    the GPU race on that array.  Output tensors may be passed in to avoid allocating
    them here too.  Returns (dq, dk, dv)."""
    _check(q, "q")
    _check_kv(q, k, v, packed=False)
    B, Sq, Hq, d = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_bwd_tensors(q, k, v, o, lse, dout, dq, dk, dv, (B, Hq, Sq))
    with torch.cuda.device(q.device):
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
    """Forward unit order: FA_SCHED_STATIC (persistent grid, fixed stride),
    FA_SCHED_CLC (one CTA per unit, running CTAs cancel pending ones to take their
    units) or FA_SCHED_AUTO (the default: CLC for causal launches over >= 4096 keys,
    else STATIC).  Process-wide."""
    _raise(_lib.load().fa_set_unit_schedule(int(mode)), "fa_set_unit_schedule")


def fa_set_exp2_emulation(pairs_of_4: int):
    """Forward exp2 split: how many of every four pairs of exponentials of an unmasked
    score tile use the FMA-pipe cubic instead of the special-function unit (0..3), or
    -1 for the library's per-head-dim default.  Process-wide."""
    _raise(_lib.load().fa_set_exp2_emulation(int(pairs_of_4)), "fa_set_exp2_emulation")


def fa_set_wait_timeout_ms(ms: int):
    """Limit (ms, 1..600000; 1000 initially) after which a kernel's pipeline wait gives
    up and reports FA_ERR_DEVICE_TIMEOUT.  Wall-clock time on the device: raise it on
    GPUs time-sliced between processes.  Process-wide."""
    _raise(_lib.load().fa_set_wait_timeout_ms(int(ms)), "fa_set_wait_timeout_ms")


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
