"""ctypes binding to libfa.so (argument marshalling only; all work runs in the kernels)."""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfa.so")

(FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_DEVICE_TIMEOUT,
 FA_ERR_SCRATCH_LIMIT) = range(6)
FA_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024
FA_BF16, FA_FP16 = 0, 1

# Every symbol include/fa.h declares, with its ctypes signature.
_vp = ctypes.c_void_p
_ci = ctypes.c_int
_cf = ctypes.c_float
_sz = ctypes.c_size_t
SIGNATURES = {
    "fa_fwd": (_ci, [_vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, _ci, _cf, _ci, _vp]),
    "fa_fwd_splitkv_workspace_size": (_sz, [_ci, _ci, _ci, _ci, _ci, _ci, _ci]),
    "fa_fwd_splitkv": (_ci, [_vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, _ci, _cf, _ci, _ci, _vp,
                             _sz, _vp]),
    "fa_fwd_varlen": (_ci, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, _ci,
                            _ci, _ci, _cf, _ci, _vp]),
    "fa_bwd_workspace_size": (_sz, [_ci, _ci, _ci, _ci]),
    "fa_bwd": (_ci, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci,
                     _ci, _cf, _ci, _vp, _sz, _vp]),
    "fa_bwd_varlen": (_ci, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci,
                            _ci, _ci, _ci, _ci, _ci, _ci, _cf, _ci, _vp, _sz, _vp]),
    "fa_bwd_noalloc": (_ci, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci,
                             _ci, _ci, _ci, _cf, _ci, _vp]),
    "fa_status_string": (ctypes.c_char_p, [_ci]),
    "fa_last_device_status": (_ci, [_vp, ctypes.POINTER(ctypes.c_uint32)]),
    "fa_clear_device_status": (_ci, [_vp]),
    "fa_debug_inject": (_ci, [_ci]),
    "fa_set_unit_schedule": (_ci, [_ci]),
    "fa_set_exp2_emulation": (_ci, [_ci]),
    "fa_set_wait_timeout_ms": (_ci, [_ci]),
    "fa_debug_exp2": (_ci, [_vp, _vp, _ci, _ci, _vp]),
}

_lock = threading.Lock()
_lib = None


def load() -> ctypes.CDLL:
    """Load libfa.so from the package directory.  Raises if it is missing: there is
    no other implementation to fall back to."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"libfa.so not found at {LIB_PATH}; build it with "
                    "`python -m exact_attention_blackwell_fa_b200.build`")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib
