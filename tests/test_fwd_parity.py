"""GPU parity of fa_fwd against the fp64 oracle (element by element).

Tolerances: O max abs error <= 1e-2 and mean abs error <= 1e-3, LSE abs error
<= 1e-3, on 16-bit inputs drawn N(0, 1) (0.5 N(0, 1) for the video shapes).
Rows that see no key (causal with Sq > Sk) must give O = 0 and LSE = -inf.
"""
import math

import pytest
import torch

from exact_attention_blackwell_fa_b200.inputs import Shape, make_inputs, sample_rows

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_MAX = 1e-2, 1e-3, 1e-3


def run_fwd(shape, causal, dtype=torch.bfloat16, amp=1.0, seed=0, scale=None):
    import exact_attention_blackwell_fa_b200 as fa

    q, k, v = make_inputs(shape, seed=seed, dtype=dtype, amp=amp)
    o, lse = fa.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale)
    torch.cuda.synchronize()
    return (q, k, v), o.cpu(), lse.cpu()


def p_rounding_bound(v, dtype):
    """Largest O error the 16-bit rounding of P alone can cause: P is rounded to the
    input dtype before the P V product (unit roundoff u = 2^-8 for bf16, 2^-11 for
    fp16), so |dO_i| <= u * sum_j P_ij |v_j| <= u * max |v|.  Used where the scale
    differs from 1/sqrt(d), which sharpens the softmax beyond the N(0, 1) tolerance."""
    u = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -11
    return u * v.double().abs().max().item() + 1e-3


def half_ulp(ref, dtype):
    """Half a unit in the last place of the 16-bit output dtype at the reference value:
    the error of rounding the exact result to the output tensor's dtype."""
    mant = 8 if dtype == torch.bfloat16 else 11          # significand bits incl. hidden
    tiny = torch.finfo(dtype).tiny
    e = torch.floor(torch.log2(ref.abs().clamp_min(tiny)))
    return torch.ldexp(torch.ones_like(ref), (e - mant).to(torch.int32))


def assert_o_close(o, o_ref, dtype, o_max=O_MAX):
    """The O bound applies to the computed result before its final rounding to the
    16-bit output: |o - o_ref| <= o_max + half an output ulp at o_ref, elementwise."""
    err = (o.double() - o_ref).abs()
    assert torch.isfinite(o.double()).all()
    excess = (err - (o_max + half_ulp(o_ref, dtype))).max().item()
    assert excess <= 0.0, f"O max abs err {err.max().item()} (excess {excess})"
    assert err.mean().item() <= O_MEAN, f"O mean abs err {err.mean().item()}"
    return err


def check_full(oracle_mod, shape, causal, dtype=torch.bfloat16, amp=1.0, scale=None):
    (q, k, v), o, lse = run_fwd(shape, causal, dtype, amp, scale=scale)
    o_ref, lse_ref = oracle_mod.fwd(q, k, v, causal=causal, scale=scale)
    o_max = O_MAX if scale is None else max(O_MAX, p_rounding_bound(v, dtype))
    err = assert_o_close(o, o_ref, dtype, o_max)
    fin = torch.isfinite(lse_ref)
    assert torch.equal(torch.isfinite(lse), fin), "LSE -inf pattern differs"
    if fin.any():
        lerr = (lse.double()[fin] - lse_ref[fin]).abs().max().item()
        assert lerr <= LSE_MAX, f"LSE abs err {lerr}"
    assert torch.all(torch.isneginf(lse[~fin]))
    return err.max().item()


SMALL = [
    # B, Sq, Sk, Hq, Hkv, d
    (1, 256, 256, 2, 2, 128),      # the small forward configuration
    (2, 384, 384, 2, 2, 128),
    (1, 300, 200, 4, 2, 128),      # ragged tails, Sq != Sk, GQA
    (1, 200, 333, 4, 1, 128),
    (1, 256, 256, 2, 2, 256),
    (2, 300, 520, 2, 1, 256),
    (1, 1, 1, 1, 1, 128),
    (1, 1, 1, 1, 1, 256),
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SMALL)
def test_fwd_small_bf16(oracle_mod, shape, causal):
    check_full(oracle_mod, Shape(*shape), causal)


@pytest.mark.parametrize("d", [128, 256])
def test_fwd_fp16(oracle_mod, d):
    check_full(oracle_mod, Shape(1, 320, 320, 2, 2, d), True, dtype=torch.float16)
    check_full(oracle_mod, Shape(1, 320, 320, 2, 2, d), False, dtype=torch.float16)


@pytest.mark.parametrize("d", [128, 256])
def test_fwd_causal_rows_without_keys(oracle_mod, d):
    """Causal with Sq much larger than Sk: whole units see no key at all."""
    check_full(oracle_mod, Shape(1, 700, 100, 2, 1, d), True)


def test_fwd_video_small(oracle_mod):
    """[1, 257, 8, 128] video-diffusion shape, inputs 0.5 N(0, 1)."""
    check_full(oracle_mod, Shape(1, 257, 257, 8, 8, 128), False, amp=0.5)


def test_fwd_custom_scale(oracle_mod):
    check_full(oracle_mod, Shape(1, 256, 384, 2, 2, 128), False, scale=0.3)
    check_full(oracle_mod, Shape(1, 256, 384, 2, 2, 256), True, scale=0.05)


def test_fwd_many_units_persistent(oracle_mod):
    """More work units than SMs so each persistent CTA walks several units."""
    shape = Shape(2, 1024, 1024, 96, 24, 128)          # 2*96*4 = 768 units
    (q, k, v), o, lse = run_fwd(shape, True)
    rows = sample_rows(2, 96, 1024, 6, seed=5)
    o_ref, lse_ref = oracle_mod.fwd(q, k, v, causal=True, rows=rows)
    got = o[rows[:, 0], rows[:, 2], rows[:, 1]].double()
    assert_o_close(got, o_ref, torch.bfloat16)
    lerr = (lse[rows[:, 0], rows[:, 1], rows[:, 2]].double() - lse_ref).abs().max().item()
    assert lerr <= LSE_MAX


def _growing_keys(shape, upper_half_only, dtype=torch.bfloat16):
    """Keys whose norm grows along the sequence, so the running row maximum keeps
    jumping by more than the rescale threshold from one KV tile to the next.  With
    upper_half_only, only keys in columns 64..127 of each 128-key tile grow, so one
    half-row's maximum jumps while the other's does not."""
    q, k, v = make_inputs(shape, seed=7, dtype=dtype)
    Sk = shape.Sk
    gain = torch.linspace(0.2, 12.0, Sk)
    if upper_half_only:
        gain = torch.where((torch.arange(Sk) % 128) >= 64, gain, torch.full_like(gain, 0.2))
    k = (k.float() * gain.view(1, Sk, 1, 1)).to(dtype)
    return q, k, v


@pytest.mark.parametrize("upper_half_only", [False, True])
@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_rescale_paths(oracle_mod, upper_half_only, d, causal):
    """Exercise the thresholded O rescale, including a reference jump seen by only one
    of the two half-row warpgroups.  These keys are far from N(0, 1) and make most rows
    attend to one or two keys, so the bound is the one the arithmetic fixes rather than
    the N(0, 1) tolerance: P is rounded to bf16 (unit roundoff u = 2^-8) before P V,
    giving |dO_i| <= u * sum_j P_ij |v_j| <= u * max |v| per element (plus the output
    rounding) and about u * mean |v| on average."""
    import exact_attention_blackwell_fa_b200 as fa

    shape = Shape(1, 256, 1024, 2, 2, d)
    q, k, v = _growing_keys(shape, upper_half_only)
    o, lse = fa.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle_mod.fwd(q, k, v, causal=causal)
    err = (o.cpu().double() - o_ref).abs()
    assert torch.isfinite(err).all()
    bound = p_rounding_bound(v, torch.bfloat16) + half_ulp(o_ref, torch.bfloat16)
    assert (err - bound).max().item() <= 0.0, f"O max abs err {err.max().item()}"
    assert err.mean().item() <= 2.0 ** -8 * v.double().abs().mean().item(), err.mean().item()
    fin = torch.isfinite(lse_ref)
    assert (lse.cpu().double()[fin] - lse_ref[fin]).abs().max().item() <= LSE_MAX * max(
        1.0, lse_ref[fin].abs().max().item() / 100.0)
