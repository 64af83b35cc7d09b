"""Split-KV forward (decode-shaped calls: few query rows over long key sequences).
The key range of each (batch, head, query block) is cut into slices computed by
separate CTAs and merged with their log-sum-exps; the result must be the plain
definition's, checked against the oracle on every row, for explicit and automatic
slice counts, with slices left empty by the causal mask, with and without pack GQA.
"""
import pytest
import torch

from exact_attention_blackwell_fa_b200.inputs import Shape, make_inputs

O_MAX, O_MEAN, LSE_MAX = 1e-2, 1e-3, 1e-3
FA_ERR_INVALID_ARG = 1


def _half_ulp(ref):
    e = torch.floor(torch.log2(ref.abs().clamp_min(torch.finfo(torch.bfloat16).tiny)))
    return torch.ldexp(torch.ones_like(ref), (e - 8).to(torch.int32))


@pytest.fixture(scope="module")
def lib():
    from exact_attention_blackwell_fa_b200 import _lib, build

    build.build()
    return _lib.load()


def test_splitkv_workspace_size(lib):
    # float32 partial O and LSE per slice and row, each part rounded to 256 bytes
    r256 = lambda x: (x + 255) // 256 * 256
    for (B, Sq, Sk, Hq, Hkv, d, s) in [(2, 1, 4096, 16, 2, 128, 8), (1, 7, 100, 4, 4, 256, 3),
                                       (3, 5, 1000, 8, 2, 192, 4), (1, 3, 900, 4, 2, 512, 3),
                                       (2, 2, 700, 2, 1, 384, 2)]:
        rows = s * B * Hq * Sq
        assert lib.fa_fwd_splitkv_workspace_size(B, Sq, Sk, Hq, Hkv, d, s) == r256(rows * d * 4) + r256(rows * 4)
    assert lib.fa_fwd_splitkv_workspace_size(1, 1, 1, 3, 2, 128, 2) == 0   # Hq % Hkv
    assert lib.fa_fwd_splitkv_workspace_size(1, 1, 1, 2, 2, 320, 2) == 0   # head dim


def test_splitkv_rejections(lib):
    F = 1 << 20
    call = lambda **kw: lib.fa_fwd_splitkv(F, F, F, F, F, 1, 1, 4096, 2, 2, 128, 0, 0.088, 0, kw.get("s", 4),
                                           kw.get("ws", F), kw.get("wsb", 1 << 30), None)
    assert call(s=65) == FA_ERR_INVALID_ARG
    assert call(ws=None) == FA_ERR_INVALID_ARG
    assert call(ws=F + 64) == FA_ERR_INVALID_ARG       # not 256-byte aligned
    assert call(wsb=16) == FA_ERR_INVALID_ARG          # too small


CASES = [
    # B, Sq, Sk, Hq, Hkv, splits
    (2, 1, 5000, 16, 2, 0),       # decode, pack GQA, automatic slices
    (2, 1, 5000, 16, 2, 7),
    (1, 16, 8192, 8, 8, 16),      # no packing
    (1, 3, 300, 4, 1, 64),        # more slices than KV tiles: empty slices
    (2, 130, 1000, 8, 2, 5),      # several query blocks
]


@pytest.mark.gpu
@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", CASES)
def test_splitkv_parity(oracle_mod, case, causal, d):
    import exact_attention_blackwell_fa_b200 as fa

    B, Sq, Sk, Hq, Hkv, splits = case
    q, k, v = make_inputs(Shape(B, Sq, Sk, Hq, Hkv, d), seed=Sq + splits)
    o, lse = fa.fa_fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=causal, num_splits=splits)
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
