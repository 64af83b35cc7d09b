"""Host-side contract of the C ABI (no GPU needed).

The library must build, load, and export every function include/fa.h declares, and
every invalid argument must come back as a status code before any CUDA call is
made ("h3-blackwell-runtime/FLASH4.md", section "API": any violation raises an
error instead of changing kernels).
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_DEVICE_TIMEOUT = range(5)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from exact_attention_blackwell_fa_b200 import _lib, build

    build.build()
    return _lib.load()


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_status_string",
              "fa_last_device_status", "fa_clear_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from exact_attention_blackwell_fa_b200 import _lib

    for name in declared_functions():
        assert hasattr(lib, name), f"libfa.so does not export {name}"
        assert name in _lib.SIGNATURES, f"binding has no signature for {name}"


def test_status_strings(lib):
    for code in range(5):
        s = lib.fa_status_string(code).decode()
        assert s.startswith("FA_")
    assert lib.fa_status_string(99).decode() == "unknown fa_status"


FAKE = 1 << 20  # 16-byte-aligned non-null host value; never dereferenced


def fwd_call(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Sq=128, Sk=128, Hq=2, Hkv=2,
             d=128, causal=0, scale=0.088, dt=0, stream=None)
    a.update(kw)
    return lib.fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Sq"], a["Sk"],
                      a["Hq"], a["Hkv"], a["d"], a["causal"], a["scale"], a["dt"], a["stream"])


def bwd_call(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, do=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, B=1,
             Sq=128, Sk=128, Hq=2, Hkv=2, d=128, causal=0, scale=0.088, dt=0, ws=FAKE,
             ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return lib.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["do"], a["dq"], a["dk"],
                      a["dv"], a["B"], a["Sq"], a["Sk"], a["Hq"], a["Hkv"], a["d"], a["causal"],
                      a["scale"], a["dt"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("call", [fwd_call, bwd_call])
@pytest.mark.parametrize("kw,code", [
    (dict(q=None), FA_ERR_INVALID_ARG),
    (dict(k=None), FA_ERR_INVALID_ARG),
    (dict(lse=None), FA_ERR_INVALID_ARG),
    (dict(B=0), FA_ERR_INVALID_ARG),
    (dict(Sq=0), FA_ERR_INVALID_ARG),
    (dict(Sk=-3), FA_ERR_INVALID_ARG),
    (dict(Hq=0), FA_ERR_INVALID_ARG),
    (dict(Hkv=0), FA_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), FA_ERR_INVALID_ARG),
    (dict(scale=0.0), FA_ERR_INVALID_ARG),
    (dict(scale=-1.0), FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), FA_ERR_INVALID_ARG),
    (dict(d=64), FA_ERR_UNSUPPORTED),
    (dict(d=320), FA_ERR_UNSUPPORTED),
    (dict(d=1024), FA_ERR_UNSUPPORTED),
    (dict(dt=2), FA_ERR_UNSUPPORTED),
    (dict(q=FAKE + 2), FA_ERR_INVALID_ARG),
    (dict(v=FAKE + 8), FA_ERR_INVALID_ARG),
    (dict(B=1 << 16, Sq=1 << 16, Hq=1 << 4, Hkv=1 << 4), FA_ERR_INVALID_ARG),
])
def test_invalid_arguments_rejected_before_any_cuda_call(lib, call, kw, code):
    assert call(lib, **kw) == code


def test_bwd_specific_rejections(lib):
    assert bwd_call(lib, do=None) == FA_ERR_INVALID_ARG
    assert bwd_call(lib, ws=None) == FA_ERR_INVALID_ARG
    assert bwd_call(lib, ws=FAKE + 16) == FA_ERR_INVALID_ARG       # not 256-byte aligned
    need = lib.fa_bwd_workspace_size(1, 128, 2, 128)
    assert bwd_call(lib, ws_bytes=need - 1) == FA_ERR_INVALID_ARG


def test_workspace_size(lib):
    # D and LSE*log2(e) (fp32 per padded row) plus the fp32 dQ accumulator
    def expect(B, Sq, Hq, d):
        r256 = lambda x: (x + 255) // 256 * 256
        rows = B * Hq * ((Sq + 127) // 128 * 128)
        return 2 * r256(rows * 4) + r256(rows * d * 4)

    for args in [(1, 1, 1, 128), (2, 16384, 16, 128), (1, 257, 8, 256), (3, 129, 5, 128), (2, 300, 4, 192)]:
        assert lib.fa_bwd_workspace_size(*args) == expect(*args)
    assert lib.fa_bwd_workspace_size(0, 10, 1, 128) == 0


def test_debug_inject_validates_mode(lib):
    assert lib.fa_debug_inject(7) == FA_ERR_INVALID_ARG
    assert lib.fa_debug_inject(0) == FA_OK


def test_valid_arguments_reach_the_device_check(lib):
    """With valid arguments and no usable GPU here, the call stops at the device
    query (FA_ERR_CUDA); on a non-sm_100 GPU it would be FA_ERR_UNSUPPORTED."""
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert fwd_call(lib) in (FA_ERR_CUDA, FA_ERR_UNSUPPORTED)


def test_python_binding_refuses_cpu_tensors():
    import torch

    import exact_attention_blackwell_fa_b200 as fa

    q = torch.zeros(1, 8, 1, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.fa_fwd(q, q, q)


def test_exp2_emulation_setting_validated(lib):
    for k in (-1, 0, 1, 2, 3):
        assert lib.fa_set_exp2_emulation(k) == FA_OK
    for k in (-2, 4, 100):
        assert lib.fa_set_exp2_emulation(k) == FA_ERR_INVALID_ARG
    assert lib.fa_set_exp2_emulation(-1) == FA_OK


def test_wide_head_dims_reach_the_device_check(lib):
    """head_dim 384 and 512 are valid forward and backward arguments (the call stops
    at the device query here, with no usable GPU)."""
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    for d in (384, 512):
        assert fwd_call(lib, d=d) in (FA_ERR_CUDA, FA_ERR_UNSUPPORTED)
        assert bwd_call(lib, d=d) in (FA_ERR_CUDA, FA_ERR_UNSUPPORTED)


def test_wait_timeout_setting_validated(lib):
    for ms in (1, 50, 1000, 600000):
        assert lib.fa_set_wait_timeout_ms(ms) == FA_OK
    for ms in (0, -5, 600001):
        assert lib.fa_set_wait_timeout_ms(ms) == FA_ERR_INVALID_ARG
    assert lib.fa_set_wait_timeout_ms(1000) == FA_OK
