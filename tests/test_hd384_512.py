"""head_dim 384 and 512 ("[RFC] FA4 -- head_dim=256 & head_dim=512", Phase 4: symmetric
head_dim=384 and head_dim=512 on SM100): forward and backward against the fp64 oracle,
element by element, at the tolerances of the other head dims (O max abs <= 1e-2 + half
an output ulp, mean <= 1e-3; LSE <= 1e-3; each gradient max abs <= 5e-2 x its largest
oracle magnitude).

At these widths a row's fp32 O accumulator does not fit in tensor memory beside the
score buffers, so each 128-row Q tile is computed by two work units, each producing one
half of O's head dims from S = Q K^T over all of them; the backward likewise runs each
64-key block as two units, one per half of the output head dims, each recomputing S and
dP over all dims in two phases.  The cases below cover both halves, ragged tiles, GQA,
rows that see no key, split KV, pack GQA and packed variable-length batches.
"""
import pytest
import torch

from exact_attention_blackwell_fa_b200.inputs import Shape, make_inputs, sample_rows

from test_hd192 import _assert_fwd, _assert_grads

pytestmark = pytest.mark.gpu

FWD = [
    # B, Sq, Sk, Hq, Hkv
    (1, 256, 256, 2, 2),
    (2, 300, 520, 4, 2),     # ragged tails, Sq != Sk, GQA
    (1, 520, 300, 2, 1),     # causal: rows that see no key
    (1, 1, 1, 1, 1),
    (1, 129, 1000, 3, 1),
]


@pytest.mark.parametrize("d", [384, 512])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("shape", FWD)
def test_wide_fwd(oracle_mod, shape, causal, dtype, d):
    import exact_attention_blackwell_fa_b200 as fa

    s = Shape(*shape, d)
    q, k, v = make_inputs(s, seed=1, dtype=dtype)
    o, lse = fa.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    o_ref, lse_ref = oracle_mod.fwd(q, k, v, causal=causal)
    _assert_fwd(o.cpu(), lse.cpu(), o_ref, lse_ref, dtype)


@pytest.mark.parametrize("d", [384, 512])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape,splits", [((2, 1, 5000, 8, 2), 0), ((1, 7, 3000, 4, 4), 5),
                                          ((1, 64, 2048, 16, 2), 0)])
def test_wide_splitkv_and_pack(oracle_mod, shape, splits, causal, d):
    import exact_attention_blackwell_fa_b200 as fa

    s = Shape(*shape, d)
    q, k, v = make_inputs(s, seed=3)
    o, lse = fa.fa_fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=causal, num_splits=splits)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    o_ref, lse_ref = oracle_mod.fwd(q, k, v, causal=causal)
    _assert_fwd(o.cpu(), lse.cpu(), o_ref, lse_ref)
    o2, lse2 = fa.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal)  # pack GQA when it applies
    torch.cuda.synchronize()
    _assert_fwd(o2.cpu(), lse2.cpu(), o_ref, lse_ref)


@pytest.mark.parametrize("d", [384, 512])
@pytest.mark.parametrize("causal", [False, True])
def test_wide_varlen(oracle_mod, causal, d):
    import exact_attention_blackwell_fa_b200 as fa

    lens_q, lens_k, H = [300, 1, 129, 640], [200, 77, 129, 700], 4
    tq, tk = sum(lens_q), sum(lens_k)
    q = make_inputs(Shape(1, tq, tq, H, H, d), seed=4)[0][0]
    k, v = (t[0] for t in make_inputs(Shape(1, tk, tk, H, H, d), seed=5)[1:])
    cq = torch.tensor([0] + list(torch.tensor(lens_q).cumsum(0)), dtype=torch.int32)
    ck = torch.tensor([0] + list(torch.tensor(lens_k).cumsum(0)), dtype=torch.int32)
    o, lse = fa.fa_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cq.cuda(), ck.cuda(), max(lens_q), max(lens_k),
                              causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    for s in range(len(lens_q)):
        a, b = int(cq[s]), int(cq[s + 1])
        c, e = int(ck[s]), int(ck[s + 1])
        o_ref, lse_ref = oracle_mod.fwd(q[a:b][None], k[c:e][None], v[c:e][None], causal=causal)
        _assert_fwd(o[a:b].cpu()[None], lse[:, a:b].cpu()[None], o_ref, lse_ref)


@pytest.mark.parametrize("d", [384, 512])
def test_wide_exp2_split(oracle_mod, d):
    import exact_attention_blackwell_fa_b200 as fa

    s = Shape(1, 400, 700, 2, 2, d)
    q, k, v = make_inputs(s, seed=9)
    o_ref, lse_ref = oracle_mod.fwd(q, k, v, causal=True)
    try:
        fa.fa_set_exp2_emulation(3)
        o, lse = fa.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
        torch.cuda.synchronize()
    finally:
        fa.fa_set_exp2_emulation(-1)
    _assert_fwd(o.cpu(), lse.cpu(), o_ref, lse_ref)


@pytest.mark.parametrize("d", [384, 512])
def test_wide_full_size_sampled(oracle_mod, d):
    """B=1, S=16384, 8 heads (about 32k tokens of work per head pair): sampled rows."""
    import exact_attention_blackwell_fa_b200 as fa

    s = Shape(1, 16384, 16384, 8, 8, d)
    q, k, v = make_inputs(s, seed=7)
    o, lse = fa.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=False)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    rows = sample_rows(s.B, s.Hq, s.Sq, 2, seed=8)
    o_ref, lse_ref = oracle_mod.fwd(q, k, v, causal=False, rows=rows)
    b, h, i = (rows[:, c].cuda() for c in range(3))
    _assert_fwd(o[b, i, h].cpu(), lse[b, h, i].cpu(), o_ref, lse_ref)


BWD = [
    (1, 256, 256, 2, 2),
    (2, 300, 200, 4, 2),     # ragged, Sq > Sk (causal: rows that see no key), GQA
    (1, 200, 333, 2, 1),
    (1, 1, 1, 1, 1),
]


@pytest.mark.parametrize("d", [384, 512])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", BWD)
def test_wide_bwd(oracle_mod, shape, causal, d):
    import exact_attention_blackwell_fa_b200 as fa

    s = Shape(*shape, d)
    q, k, v, do = make_inputs(s, seed=2, with_dout=True)
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.fa_fwd(qc, kc, vc, causal=causal)
    dq, dk, dv = fa.fa_bwd(qc, kc, vc, o, lse, doc, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    rq, rk, rv, _ = oracle_mod.bwd(q, k, v, do, causal=causal)
    _assert_grads((dq.cpu(), dk.cpu(), dv.cpu()), (rq, rk, rv))


@pytest.mark.parametrize("d", [384, 512])
def test_wide_bwd_fp16(oracle_mod, d):
    import exact_attention_blackwell_fa_b200 as fa

    s = Shape(1, 320, 320, 2, 2, d)
    q, k, v, do = make_inputs(s, seed=12, dtype=torch.float16, with_dout=True)
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.fa_fwd(qc, kc, vc, causal=True)
    dq, dk, dv = fa.fa_bwd(qc, kc, vc, o, lse, doc, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    rq, rk, rv, _ = oracle_mod.bwd(q, k, v, do, causal=True)
    _assert_grads((dq.cpu(), dk.cpu(), dv.cpu()), (rq, rk, rv))


@pytest.mark.parametrize("d", [384, 512])
@pytest.mark.parametrize("causal", [False, True])
def test_wide_bwd_varlen(oracle_mod, causal, d):
    import exact_attention_blackwell_fa_b200 as fa

    lens_q, lens_k, H = [300, 1, 129, 640], [200, 77, 129, 700], 4
    tq, tk = sum(lens_q), sum(lens_k)
    q = make_inputs(Shape(1, tq, tq, H, H, d), seed=4)[0][0]
    k, v = (t[0] for t in make_inputs(Shape(1, tk, tk, H, H, d), seed=5)[1:])
    do = make_inputs(Shape(1, tq, tq, H, H, d), seed=6, with_dout=True)[3][0]
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
        rq, rk, rv, _ = oracle_mod.bwd(qs, ks, vs, dos, causal=causal)
        _assert_grads((dq[a:b].cpu()[None], dk[c:e].cpu()[None], dv[c:e].cpu()[None]), (rq, rk, rv))


@pytest.mark.parametrize("d", [384, 512])
def test_wide_bwd_full_size_sampled(oracle_mod, d):
    """B=1, S=8192, 8 heads: dQ on sampled query rows, dK / dV on sampled keys of the
    first and last KV heads (both output halves of every key row)."""
    import exact_attention_blackwell_fa_b200 as fa

    s = Shape(1, 8192, 8192, 8, 8, d)
    q, k, v, do = make_inputs(s, seed=17, with_dout=True)
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.fa_fwd(qc, kc, vc, causal=True)
    dq, dk, dv = fa.fa_bwd(qc, kc, vc, o, lse, doc, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    qrows = sample_rows(s.B, s.Hq, s.Sq, 2, seed=9)
    js = torch.tensor([0, 1, 4095, 8191])
    kvrows = torch.cat([torch.stack([torch.zeros_like(js), torch.full_like(js, h), js], 1) for h in (0, s.Hkv - 1)])
    rq, rk, rv, _ = oracle_mod.bwd(q, k, v, do, causal=True, qrows=qrows, kvrows=kvrows)
    qb, qh, qi = (qrows[:, c].cuda() for c in range(3))
    kb, kh, kj = (kvrows[:, c].cuda() for c in range(3))
    _assert_grads((dq[qb, qi, qh].cpu(), dk[kb, kj, kh].cpu(), dv[kb, kj, kh].cpu()), (rq, rk, rv))
