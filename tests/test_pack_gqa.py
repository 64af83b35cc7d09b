"""Pack GQA ("[RFC] FA4 -- head_dim=256 & head_dim=512", pack_gqa row): with fewer than
256 queries per head and a power-of-two group of up to 16 query heads per KV head,
the forward fills each 128-row Q tile with the group's heads together (row r of a
(batch, KV head) = query r / group of head kv_head * group + r % group), one K/V
stream serving the whole group.  The result must be the plain definition's, so these
cases are checked against the oracle on every row, including decode-shaped ones
(Sq = 1) and ragged ones, causal (bottom-right aligned) and not.
"""
import pytest
import torch

from exact_attention_blackwell_fa_b200.inputs import Shape, make_inputs

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_MAX = 1e-2, 1e-3, 1e-3


def _half_ulp(ref):
    e = torch.floor(torch.log2(ref.abs().clamp_min(torch.finfo(torch.bfloat16).tiny)))
    return torch.ldexp(torch.ones_like(ref), (e - 8).to(torch.int32))


def check(oracle_mod, shape, causal, seed=0):
    import exact_attention_blackwell_fa_b200 as fa

    q, k, v = make_inputs(shape, seed=seed)
    o, lse = fa.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    o_ref, lse_ref = oracle_mod.fwd(q, k, v, causal=causal)
    err = (o.cpu().double() - o_ref).abs()
    assert (err - (O_MAX + _half_ulp(o_ref))).max().item() <= 0.0, err.max().item()
    assert err.mean().item() <= O_MEAN
    lg = lse.cpu().double()
    fin = torch.isfinite(lse_ref)
    assert torch.equal(torch.isfinite(lg), fin)
    if fin.any():
        assert (lg[fin] - lse_ref[fin]).abs().max().item() <= LSE_MAX


CASES = [
    # B, Sq, Sk, Hq, Hkv
    (2, 1, 1000, 16, 2),      # decode, group 8
    (1, 3, 517, 16, 1),       # group 16
    (2, 17, 300, 8, 2),       # group 4, ragged
    (1, 64, 1024, 8, 4),      # group 2
    (1, 200, 200, 16, 4),     # group 4, 800 packed rows (several units)
    (1, 255, 90, 4, 2),       # more queries than keys
    (1, 5, 1, 8, 1),          # one key
    (1, 9, 400, 6, 2),        # group 3: not packed
]


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", CASES)
def test_pack_gqa_parity(oracle_mod, case, causal, d):
    B, Sq, Sk, Hq, Hkv = case
    check(oracle_mod, Shape(B, Sq, Sk, Hq, Hkv, d), causal, seed=Sq)
