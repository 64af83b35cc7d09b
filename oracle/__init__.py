"""fp64 CPU oracle for exact scaled-dot-product attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  It is independent of the CUDA library: it shares no
code with it and never imports it.  The arithmetic lives in ``attn_oracle.c``
(plain C, double precision, OpenMP over independent rows); this module only
compiles that file and marshals tensors into it.

Definition followed (one query row at a time, full score row, no tiling):
``O = softmax(scale * Q K^T [+ causal mask]) V`` and ``LSE = M + ln(l)`` as in
"FlashAttention 4: Snellere, Geheugenefficiente Aandacht voor LLM's",
introduction and section "Slimmere Online Softmax-herwaardering"; the backward
is the explicit chain rule of that definition (see the header of the C file).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_attn.so")
_lock = threading.Lock()
_lib = None

BF16, FP16, F64 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into liboracle_attn.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64p = ctypes.POINTER(ctypes.c_int64)
            dp = ctypes.POINTER(ctypes.c_double)
            vp = ctypes.c_void_p
            ci = ctypes.c_int
            lib.fa_oracle_fwd.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, ci,
                                          ctypes.c_double, i64p, ctypes.c_int64, dp, dp]
            lib.fa_oracle_fwd.restype = ci
            lib.fa_oracle_bwd.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, ci,
                                          ctypes.c_double, i64p, ctypes.c_int64, dp, dp,
                                          i64p, ctypes.c_int64, dp, dp]
            lib.fa_oracle_bwd.restype = ci
            lib.fa_oracle_num_threads.argtypes = []
            lib.fa_oracle_num_threads.restype = ci
            _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().fa_oracle_num_threads())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float16:
        return FP16
    if t.dtype == torch.float64:
        return F64
    raise TypeError(f"oracle takes bf16/fp16 (or float64) inputs, got {t.dtype}")


def _host16(t: torch.Tensor) -> torch.Tensor:
    return t.detach().to("cpu").contiguous()


def _rows(rows, default_fn) -> torch.Tensor:
    if rows is None:
        rows = default_fn()
    r = torch.as_tensor(rows, dtype=torch.int64).reshape(-1, 3).contiguous()
    return r


def _ptr(t: torch.Tensor, ty):
    return ctypes.cast(t.data_ptr(), ctypes.POINTER(ty)) if t.numel() else None


def all_rows(B: int, H: int, S: int) -> torch.Tensor:
    """Every (b, h, i) triple in row-major order."""
    b = torch.arange(B).view(B, 1, 1).expand(B, H, S)
    h = torch.arange(H).view(1, H, 1).expand(B, H, S)
    i = torch.arange(S).view(1, 1, S).expand(B, H, S)
    return torch.stack([b, h, i], dim=-1).reshape(-1, 3).contiguous()


def fwd(q, k, v, causal=False, scale=None, rows=None):
    """Oracle forward.

    q: [B, Sq, Hq, d], k/v: [B, Sk, Hkv, d] (bf16 or fp16, any device).
    rows: optional (n, 3) list of (b, h, i); default every row.
    Returns (o, lse) in float64: o is (n, d) for explicit rows, else [B, Sq, Hq, d];
    lse is (n,) for explicit rows, else [B, Hq, Sq].
    """
    B, Sq, Hq, d = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = d ** -0.5
    explicit = rows is not None
    r = _rows(rows, lambda: all_rows(B, Hq, Sq))
    qh, kh, vh = _host16(q), _host16(k), _host16(v)
    dt = _dtype_code(qh)
    n = r.shape[0]
    o = torch.empty(n, d, dtype=torch.float64)
    lse = torch.empty(n, dtype=torch.float64)
    rc = _load().fa_oracle_fwd(qh.data_ptr(), kh.data_ptr(), vh.data_ptr(), dt, B, Sq, Sk, Hq,
                               Hkv, d, int(bool(causal)), float(scale),
                               _ptr(r, ctypes.c_int64), n, _ptr(o, ctypes.c_double),
                               _ptr(lse, ctypes.c_double))
    if rc:
        raise RuntimeError(f"fa_oracle_fwd failed with code {rc}")
    if explicit:
        return o, lse
    return (o.view(B, Hq, Sq, d).permute(0, 2, 1, 3).contiguous(), lse.view(B, Hq, Sq))


def bwd(q, k, v, dout, causal=False, scale=None, qrows=None, kvrows=None):
    """Oracle backward.

    qrows: (n, 3) of (b, h, i) for dQ and D; kvrows: (m, 3) of (b, hkv, j) for dK, dV.
    With both None every row is computed and full tensors are returned:
    dq [B, Sq, Hq, d], dk/dv [B, Sk, Hkv, d], D [B, Hq, Sq].  With explicit lists the
    per-row arrays (n, d), (m, d), (n,) are returned.  All float64.
    """
    B, Sq, Hq, d = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = d ** -0.5
    full = qrows is None and kvrows is None
    qr = _rows(qrows, lambda: all_rows(B, Hq, Sq)) if (full or qrows is not None) else \
        torch.empty(0, 3, dtype=torch.int64)
    kr = _rows(kvrows, lambda: all_rows(B, Hkv, Sk)) if (full or kvrows is not None) else \
        torch.empty(0, 3, dtype=torch.int64)
    qh, kh, vh, dh = _host16(q), _host16(k), _host16(v), _host16(dout)
    dt = _dtype_code(qh)
    nq, nk = qr.shape[0], kr.shape[0]
    dq = torch.empty(nq, d, dtype=torch.float64)
    D = torch.empty(nq, dtype=torch.float64)
    dk = torch.empty(nk, d, dtype=torch.float64)
    dv = torch.empty(nk, d, dtype=torch.float64)
    dp = ctypes.c_double
    rc = _load().fa_oracle_bwd(qh.data_ptr(), kh.data_ptr(), vh.data_ptr(), dh.data_ptr(), dt,
                               B, Sq, Sk, Hq, Hkv, d, int(bool(causal)), float(scale),
                               _ptr(qr, ctypes.c_int64), nq, _ptr(dq, dp), _ptr(D, dp),
                               _ptr(kr, ctypes.c_int64), nk, _ptr(dk, dp), _ptr(dv, dp))
    if rc:
        raise RuntimeError(f"fa_oracle_bwd failed with code {rc}")
    if not full:
        return dq, dk, dv, D
    return (dq.view(B, Hq, Sq, d).permute(0, 2, 1, 3).contiguous(),
            dk.view(B, Hkv, Sk, d).permute(0, 2, 1, 3).contiguous(),
            dv.view(B, Hkv, Sk, d).permute(0, 2, 1, 3).contiguous(),
            D.view(B, Hq, Sq))
