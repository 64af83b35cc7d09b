"""head_dim 192 ("[RFC] FA4 -- head_dim=256 & head_dim=512", Phase 4: symmetric
head_dim=192 on SM100): forward, backward, split KV, pack GQA and packed variable-length
batches against the fp64 oracle, element by element, at the same tolerances as the
other head dims (O max abs <= 1e-2 + half an output ulp, mean <= 1e-3; LSE <= 1e-3;
each gradient max abs <= 5e-2 x its largest oracle magnitude).

The forward streams K and V through a ring of 128-row x 64-dim chunks (three per
tile); the backward runs the 64-key-unit kernel of head_dim 256 with the fourth
64-dim block of every operand tile zero, so these cases also cover the head-dim
lanes that kernel must leave unwritten.
"""
import pytest
import torch

from exact_attention_blackwell_fa_b200.inputs import Shape, make_inputs, sample_rows

pytestmark = pytest.mark.gpu

D = 192
O_MAX, O_MEAN, LSE_MAX, GRAD_REL = 1e-2, 1e-3, 1e-3, 5e-2


def _half_ulp(ref, dtype=torch.bfloat16):
    mant = 8 if dtype == torch.bfloat16 else 11
    e = torch.floor(torch.log2(ref.abs().clamp_min(torch.finfo(dtype).tiny)))
    return torch.ldexp(torch.ones_like(ref), (e - mant).to(torch.int32))


def _assert_fwd(o, lse, o_ref, lse_ref, dtype=torch.bfloat16):
    o = o.double()
    assert torch.isfinite(o).all()
    err = (o - o_ref).abs()
    excess = (err - (O_MAX + _half_ulp(o_ref, dtype))).max().item()
    assert excess <= 0.0, f"O max abs err {err.max().item():.3e}"
    assert err.mean().item() <= O_MEAN, f"O mean abs err {err.mean().item():.3e}"
    lse = lse.double()
    fin = torch.isfinite(lse_ref)
    assert torch.equal(torch.isfinite(lse), fin), "LSE -inf pattern differs"
    if fin.any():
        assert (lse[fin] - lse_ref[fin]).abs().max().item() <= LSE_MAX
    assert torch.all(torch.isneginf(lse[~fin]))


def _assert_grads(got, ref):
    big = max(r.abs().max().item() for r in ref)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        g = g.double()
        assert torch.isfinite(g).all(), name
        scale = r.abs().max().item() or big
        err = (g - r).abs().max().item()
        assert err <= GRAD_REL * scale, f"{name}: {err:.3e} > 5e-2 * {scale:.3e}"


FWD = [
    # B, Sq, Sk, Hq, Hkv
    (1, 256, 256, 2, 2),
    (2, 300, 520, 4, 2),     # ragged tails, Sq != Sk, GQA
    (1, 520, 300, 2, 1),     # causal: rows that see no key
    (1, 1, 1, 1, 1),
    (1, 129, 1000, 3, 1),
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("shape", FWD)
def test_hd192_fwd(oracle_mod, shape, causal, dtype):
    import exact_attention_blackwell_fa_b200 as fa

    s = Shape(*shape, D)
    q, k, v = make_inputs(s, seed=1, dtype=dtype)
    o, lse = fa.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    o_ref, lse_ref = oracle_mod.fwd(q, k, v, causal=causal)
    _assert_fwd(o.cpu(), lse.cpu(), o_ref, lse_ref, dtype)


BWD = [
    (1, 256, 256, 2, 2),
    (2, 300, 200, 4, 2),
    (1, 200, 333, 2, 1),
    (1, 1, 1, 1, 1),
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", BWD)
def test_hd192_bwd(oracle_mod, shape, causal):
    import exact_attention_blackwell_fa_b200 as fa

    s = Shape(*shape, D)
    q, k, v, do = make_inputs(s, seed=2, with_dout=True)
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.fa_fwd(qc, kc, vc, causal=causal)
    dq, dk, dv = fa.fa_bwd(qc, kc, vc, o, lse, doc, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    rq, rk, rv, _ = oracle_mod.bwd(q, k, v, do, causal=causal)
    _assert_grads((dq.cpu(), dk.cpu(), dv.cpu()), (rq, rk, rv))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape,splits", [((2, 1, 5000, 8, 2), 0), ((1, 7, 3000, 4, 4), 5),
                                          ((1, 64, 4096, 16, 2), 0)])
def test_hd192_splitkv_and_pack(oracle_mod, shape, splits, causal):
    import exact_attention_blackwell_fa_b200 as fa

    s = Shape(*shape, D)
    q, k, v = make_inputs(s, seed=3)
    o, lse = fa.fa_fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=causal, num_splits=splits)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    o_ref, lse_ref = oracle_mod.fwd(q, k, v, causal=causal)
    _assert_fwd(o.cpu(), lse.cpu(), o_ref, lse_ref)
    o2, lse2 = fa.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal)  # pack GQA when it applies
    torch.cuda.synchronize()
    _assert_fwd(o2.cpu(), lse2.cpu(), o_ref, lse_ref)


@pytest.mark.parametrize("causal", [False, True])
def test_hd192_varlen(oracle_mod, causal):
    import exact_attention_blackwell_fa_b200 as fa

    lens_q, lens_k, H = [300, 1, 129, 640], [200, 77, 129, 700], 4
    tq, tk = sum(lens_q), sum(lens_k)
    q = make_inputs(Shape(1, tq, tq, H, H, D), seed=4)[0][0]
    k, v = (t[0] for t in make_inputs(Shape(1, tk, tk, H, H, D), seed=5)[1:])
    do = make_inputs(Shape(1, tq, tq, H, H, D), seed=6, with_dout=True)[3][0]
    cq = torch.tensor([0] + list(torch.tensor(lens_q).cumsum(0)), dtype=torch.int32)
    ck = torch.tensor([0] + list(torch.tensor(lens_k).cumsum(0)), dtype=torch.int32)
    args = (cq.cuda(), ck.cuda(), max(lens_q), max(lens_k))
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.fa_fwd_varlen(qc, kc, vc, *args, causal=causal)
    dq, dk, dv = fa.fa_bwd_varlen(qc, kc, vc, o, lse, doc, *args, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    for s in range(len(lens_q)):
        a, b = int(cq[s]), int(cq[s + 1])
        c, e = int(ck[s]), int(ck[s + 1])
        qs, ks, vs, dos = q[a:b][None], k[c:e][None], v[c:e][None], do[a:b][None]
        o_ref, lse_ref = oracle_mod.fwd(qs, ks, vs, causal=causal)
        _assert_fwd(o[a:b].cpu()[None], lse[:, a:b].cpu()[None], o_ref, lse_ref)
        rq, rk, rv, _ = oracle_mod.bwd(qs, ks, vs, dos, causal=causal)
        _assert_grads((dq[a:b].cpu()[None], dk[c:e].cpu()[None], dv[c:e].cpu()[None]), (rq, rk, rv))


@pytest.mark.parametrize("causal", [False, True])
def test_hd192_full_size_sampled(oracle_mod, causal):
    """B=2, S=16384, 8 heads: forward rows and backward rows / keys sampled per head."""
    import exact_attention_blackwell_fa_b200 as fa

    s = Shape(2, 16384, 16384, 8, 8, D)
    q, k, v, do = make_inputs(s, seed=7, with_dout=True)
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.fa_fwd(qc, kc, vc, causal=causal)
    dq, dk, dv = fa.fa_bwd(qc, kc, vc, o, lse, doc, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    rows = sample_rows(s.B, s.Hq, s.Sq, 3, seed=8)
    o_ref, lse_ref = oracle_mod.fwd(q, k, v, causal=causal, rows=rows)
    b, h, i = (rows[:, c].cuda() for c in range(3))
    _assert_fwd(o[b, i, h].cpu(), lse[b, h, i].cpu(), o_ref, lse_ref)
    qrows = sample_rows(s.B, s.Hq, s.Sq, 2, seed=9)
    js = torch.tensor([0, 1, 8191, 16383])
    kvrows = torch.stack([torch.ones_like(js), torch.full_like(js, s.Hkv - 1), js], 1)
    rq, rk, rv, _ = oracle_mod.bwd(q, k, v, do, causal=causal, qrows=qrows, kvrows=kvrows)
    qb, qh, qi = (qrows[:, c].cuda() for c in range(3))
    kb, kh, kj = (kvrows[:, c].cuda() for c in range(3))
    _assert_grads((dq[qb, qi, qh].cpu(), dk[kb, kj, kh].cpu(), dv[kb, kj, kh].cpu()), (rq, rk, rv))
