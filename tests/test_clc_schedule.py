"""Unit order by cluster launch control ("[RFC] FA4 -- head_dim=256 & head_dim=512",
Phase 2 persistent + cluster-aware tile scheduler, Phase 3 CLC scheduling).

With FA_SCHED_CLC the forward launches one CTA per work unit and the running CTAs
take the remaining units by cancelling CTAs that have not started.  Which CTA
computes a unit does not change its arithmetic, so the outputs must equal the
static schedule's bit for bit; sampled rows are also checked against the oracle.
Shapes have more units than the 148 SMs (otherwise both modes launch the same grid).
"""
import pytest
import torch

from exact_attention_blackwell_fa_b200.inputs import Shape, make_inputs, sample_rows

O_MAX, LSE_MAX = 1e-2, 1e-3


@pytest.fixture
def clc_mode():
    import exact_attention_blackwell_fa_b200 as fa

    yield fa
    fa.fa_set_unit_schedule(fa.FA_SCHED_AUTO)


def test_schedule_mode_arguments():
    from exact_attention_blackwell_fa_b200 import _lib

    lib = _lib.load()
    assert lib.fa_set_unit_schedule(3) == 1 and lib.fa_set_unit_schedule(-1) == 1  # FA_ERR_INVALID_ARG
    assert lib.fa_set_unit_schedule(1) == 0 and lib.fa_set_unit_schedule(0) == 0
    assert lib.fa_set_unit_schedule(2) == 0  # FA_SCHED_AUTO, the default


def _both(fa, fn):
    fa.fa_set_unit_schedule(fa.FA_SCHED_STATIC)
    a = fn()
    fa.fa_set_unit_schedule(fa.FA_SCHED_CLC)
    b = fn()
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    return a, b


CASES = [
    # B, Sq, Sk, Hq, Hkv, d
    (4, 4096, 4096, 16, 16, 128),    # 1024 units
    (8, 1024, 1024, 16, 4, 128),     # GQA, 512 units
    (2, 8192, 8192, 8, 8, 256),      # 1024 units
    (16, 1000, 1300, 8, 8, 192),     # ragged tails, Sq != Sk
]


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", CASES)
def test_clc_matches_static_and_oracle(oracle_mod, clc_mode, shape, causal):
    fa = clc_mode
    s = Shape(*shape)
    q, k, v = make_inputs(s, seed=21)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    (o0, l0), (o1, l1) = _both(fa, lambda: fa.fa_fwd(qc, kc, vc, causal=causal))
    assert torch.equal(o0, o1) and torch.equal(l0, l1)
    rows = sample_rows(s.B, s.Hq, s.Sq, 2, seed=22)
    o_ref, lse_ref = oracle_mod.fwd(q, k, v, causal=causal, rows=rows)
    b, h, i = (rows[:, c].cuda() for c in range(3))
    err = (o1[b, i, h].cpu().double() - o_ref).abs().max().item()
    assert err <= O_MAX + 2.0 ** -8
    fin = torch.isfinite(lse_ref)
    got = l1[b, h, i].cpu().double()
    assert torch.equal(torch.isfinite(got), fin)
    if fin.any():
        assert (got[fin] - lse_ref[fin]).abs().max().item() <= LSE_MAX


@pytest.mark.gpu
def test_clc_splitkv_pack_and_varlen(clc_mode):
    """The other forward entry points under FA_SCHED_CLC: split KV with pack GQA
    (decode-shaped) and a packed variable-length batch; bit-equal to the static order."""
    fa = clc_mode
    q, k, v = (t.cuda() for t in make_inputs(Shape(64, 1, 8192, 32, 4, 128), seed=23))
    (o0, l0), (o1, l1) = _both(fa, lambda: fa.fa_fwd_splitkv(q, k, v, num_splits=8))
    assert torch.equal(o0, o1) and torch.equal(l0, l1)
    lens = [3000, 1, 700, 4096, 129, 2048]
    tot = sum(lens)
    qv, kv, vv = (t[0].cuda() for t in make_inputs(Shape(1, tot, tot, 16, 16, 128), seed=24))
    cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0)), dtype=torch.int32, device="cuda")
    for causal in (False, True):
        (o0, l0), (o1, l1) = _both(
            fa, lambda: fa.fa_fwd_varlen(qv, kv, vv, cu, cu, max(lens), max(lens), causal=causal))
        assert torch.equal(o0, o1) and torch.equal(l0, l1)
