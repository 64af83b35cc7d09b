"""The exp2 used by the kernels' exponential split ("Software-exponentials via
CUDA-kernen", FlashAttention 4 page: part of the exponentials computed with a cubic
on the FMA pipe instead of the SFU).  The pages give no coefficients; ours are a
relative-minimax fit (exact_attention_blackwell_fa_b200/csrc/fit_exp2_poly.py).

CPU: the committed coefficients, evaluated with the kernel's range reduction in
fp32 (x = n + f, n = round(x), f in [-1/2, 1/2], 2^n into the exponent field), stay
within 2^-9 relative of fp64 2^x over a dense grid (the bound below the 16-bit
rounding of P that the tolerances assume).
GPU: the device forms through the fa_debug_exp2 hook, against fp64 2^x.
"""
import os
import re

import numpy as np
import pytest
import torch

HDR = os.path.join(os.path.dirname(__file__), "..", "exact_attention_blackwell_fa_b200", "csrc", "exp2_poly.h")
BOUND = 2.0 ** -9


def _coeffs():
    txt = open(HDR).read()
    c = {k: float(v) for k, v in re.findall(r"#define FA_EXP2_(C\d) ([0-9.eE+-]+)f", txt)}
    return [np.float32(c[f"C{i}"]) for i in range(4)]


def _emulate(x):
    """fp32 evaluation with the kernel's steps (each operation rounded to fp32; the
    Horner steps are fused multiply-adds, emulated in fp64 and rounded once)."""
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    f64 = f.astype(np.float64)
    p = np.float32(c3 * f64 + np.float64(c2))
    p = np.float32(p.astype(np.float64) * f64 + np.float64(c1))
    p = np.float32(p.astype(np.float64) * f64 + np.float64(c0))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) & np.uint64(0xFFFFFFFF)
    return bits.astype(np.uint32).view(np.float32)


def test_range_reduction_is_exact():
    x = np.linspace(-126.0, 8.0, 200001, dtype=np.float32)
    magic = np.float32(12582912.0)
    n = ((x + magic).astype(np.float32) - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    assert np.all(np.abs(f) <= 0.5)
    assert np.array_equal(n, np.round(x))  # round half to even, like the fp32 add
    assert np.array_equal((f.astype(np.float64) + n), x.astype(np.float64))


def test_cubic_relative_error_dense_grid():
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    y = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() <= BOUND
    assert rel.max() <= 1.05 * 1.438856e-04  # the figure recorded with the coefficients


def test_cubic_integers_and_signs():
    x = np.arange(-125, 9, dtype=np.float32)
    y = _emulate(x).astype(np.float64)
    assert np.all(y > 0)
    assert np.max(np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)) <= BOUND
    # monotone on a fine grid around an integer boundary (no jump at n changes)
    xs = np.linspace(-3.6, -2.4, 4001, dtype=np.float32)
    ys = _emulate(xs)
    assert np.all(np.diff(ys.astype(np.float64)) >= -1e-6 * ys[:-1])


@pytest.mark.gpu
@pytest.mark.parametrize("mode,bound", [(0, BOUND), (1, 2.0 ** -21)])
def test_device_exp2_forms(mode, bound):
    import exact_attention_blackwell_fa_b200 as fa

    x = torch.linspace(-125.0, 8.0, 1_000_003, dtype=torch.float32, device="cuda")
    y = fa.fa_debug_exp2(x, mode=mode)
    torch.cuda.synchronize()
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel <= bound, rel
    if mode == 0:  # same fp32 steps as the CPU emulation
        emu = torch.from_numpy(_emulate(x.cpu().numpy())).cuda()
        assert ((y - emu).abs() / emu).max().item() <= 2.0 ** -22
    # far below the clamp both forms give (near) zero
    xl = torch.linspace(-400.0, -127.0, 1001, dtype=torch.float32, device="cuda")
    yl = fa.fa_debug_exp2(xl, mode=mode)
    torch.cuda.synchronize()
    assert torch.all(yl >= 0) and yl.max().item() <= 2.0 ** -125
