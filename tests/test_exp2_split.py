"""The exp2 split of the forward on the hot path, against the fp64 oracle.

fa_set_exp2_emulation(k) sends k of every four pairs of exponentials of an unmasked
score tile to the FMA-pipe cubic instead of the special-function unit ("FlashAttention
4: Snellere, Geheugenefficiente Aandacht voor LLM's", section "Software-exponentials
via CUDA-kernen"; "[RFC] FA4 -- head_dim=256 & head_dim=512", Phase 2 "exp2 FMA
emulation", 3 of 4 at head_dim 256).  The cubic's relative error (1.44e-4) is below
the 16-bit rounding of P, so the forward tolerances are unchanged: O max abs <= 1e-2
(+ half an output ulp), mean <= 1e-3, LSE abs <= 1e-3.  Shapes span several KV tiles
with a ragged tail, so unmasked tiles (split) and masked ones (SFU only) both occur.
"""
import pytest
import torch

from exact_attention_blackwell_fa_b200.inputs import Shape

from test_fwd_parity import LSE_MAX, _growing_keys, check_full, half_ulp, p_rounding_bound

pytestmark = pytest.mark.gpu


@pytest.fixture
def emu():
    import exact_attention_blackwell_fa_b200 as fa

    yield fa.fa_set_exp2_emulation
    fa.fa_set_exp2_emulation(-1)


@pytest.mark.parametrize("k", [1, 2, 3])
@pytest.mark.parametrize("d", [128, 192, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_split_matches_oracle(oracle_mod, emu, k, d, causal):
    emu(k)
    check_full(oracle_mod, Shape(1, 700, 650, 4, 2, d), causal)


@pytest.mark.parametrize("d", [128, 256])
def test_split_fp16_and_scale(oracle_mod, emu, d):
    emu(3)
    check_full(oracle_mod, Shape(1, 384, 520, 2, 2, d), False, dtype=torch.float16)
    check_full(oracle_mod, Shape(1, 256, 640, 2, 2, d), False, scale=0.3)


@pytest.mark.parametrize("d", [128, 256])
def test_split_rescale_and_wide_range(oracle_mod, emu, d):
    """Growing keys: the running maximum jumps past the rescale threshold, and most
    exponents are far below zero (the cubic's input clamp at -126 is reached)."""
    import exact_attention_blackwell_fa_b200 as fa

    emu(3)
    shape = Shape(1, 256, 1024, 2, 2, d)
    q, k, v = _growing_keys(shape, False)
    o, lse = fa.fa_fwd(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle_mod.fwd(q, k, v)
    err = (o.cpu().double() - o_ref).abs()
    bound = p_rounding_bound(v, torch.bfloat16) + half_ulp(o_ref, torch.bfloat16)
    assert (err - bound).max().item() <= 0.0, err.max().item()
    assert (lse.cpu().double() - lse_ref).abs().max().item() <= LSE_MAX * max(1.0, lse_ref.abs().max().item() / 100)


def test_split_rows_without_keys(oracle_mod, emu):
    """Causal with Sq > Sk: rows that see no key stay O = 0, LSE = -inf."""
    emu(3)
    check_full(oracle_mod, Shape(1, 700, 100, 2, 1, 128), True)
    check_full(oracle_mod, Shape(1, 700, 100, 2, 1, 256), True)
