"""The one accuracy table the pages print: FlashAttention-4 against PyTorch SDPA on the
H3 video-attention shapes, bf16 (tests/golden/gb10_validation.json, from
"h3-blackwell-runtime/FLASH4.md", section "GB10 Validation").  The page does not give
its inputs, so this is an order-of-magnitude check on the synthetic recipe for those
shapes (0.5 N(0, 1), rounded to bf16): against SDPA in bf16, the library's forward and
the oracle rounded to bf16 must both stay within twice the page's maximum difference.
Both figures are one to two bf16 units in the last place at the outputs' magnitude."""
import json
import os

import pytest
import torch
import torch.nn.functional as F

from exact_attention_blackwell_fa_b200.inputs import Shape, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "gb10_validation.json")


def _cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


def _sdpa(q, k, v):
    """PyTorch SDPA in [B, S, H, d] layout, output in the inputs' dtype."""
    o = F.scaled_dot_product_attention(q.permute(0, 2, 1, 3), k.permute(0, 2, 1, 3), v.permute(0, 2, 1, 3))
    return o.permute(0, 2, 1, 3)


def test_golden_fixture_is_the_page_table():
    c = _cases()
    assert [x["shape"] for x in c] == [[1, 257, 8, 128], [1, 20480, 56, 128]]
    assert c[0]["max_abs"] == 2.0 ** -9 and abs(c[1]["max_abs"] - 2.0 ** -12) < 1e-9


def test_oracle_rounded_to_bf16_within_page_bound(oracle_mod):
    case = _cases()[0]  # the short shape: the fp64 oracle and CPU SDPA finish in seconds
    B, S, H, d = case["shape"]
    q, k, v = make_inputs(Shape(B, S, S, H, H, d), seed=0, amp=0.5)
    o_ref, _ = oracle_mod.fwd(q, k, v)
    ref16 = o_ref.to(torch.bfloat16).double()
    sd = _sdpa(q, k, v).double()
    assert (ref16 - sd).abs().max().item() <= 2 * case["max_abs"]


@pytest.mark.gpu
@pytest.mark.parametrize("i", [0, 1])
def test_forward_against_sdpa_within_page_bound(i):
    import exact_attention_blackwell_fa_b200 as fa

    case = _cases()[i]
    B, S, H, d = case["shape"]
    q, k, v = (t.cuda() for t in make_inputs(Shape(B, S, S, H, H, d), seed=0, amp=0.5))
    o, _ = fa.fa_fwd(q, k, v)
    sd = _sdpa(q, k, v)
    torch.cuda.synchronize()
    err = (o.double() - sd.double()).abs()
    assert err.max().item() <= 2 * case["max_abs"], err.max().item()
