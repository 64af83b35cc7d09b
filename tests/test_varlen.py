"""Packed variable-length batches (cu_seqlens / seqused_k: "[RFC] FA4 -- head_dim=256
& head_dim=512", Phase 1 table).  Each sequence is an independent attention problem,
so the oracle is the plain definition applied to every sequence's slice.

Host side (no GPU): argument checks of fa_fwd_varlen.
GPU: parity against the oracle per sequence for ragged lengths (1, multiples of 128
and not, a zero-length sequence, more keys than queries and fewer), GQA, causal and
not, head_dim 128 and 256, seqused_k below the allocated key counts.
"""
import pytest
import torch

from exact_attention_blackwell_fa_b200.inputs import Shape, make_inputs

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA = range(4)
FAKE = 1 << 20
O_MAX, O_MEAN, LSE_MAX = 1e-2, 1e-3, 1e-3


@pytest.fixture(scope="module")
def lib():
    from exact_attention_blackwell_fa_b200 import _lib, build

    build.build()
    return _lib.load()


def varlen_call(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, cq=FAKE, ck=FAKE, uk=None, B=2, mq=128, mk=128,
             tq=200, tk=200, Hq=2, Hkv=2, d=128, causal=0, scale=0.088, dt=0, stream=None)
    a.update(kw)
    return lib.fa_fwd_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cq"], a["ck"], a["uk"], a["B"],
                             a["mq"], a["mk"], a["tq"], a["tk"], a["Hq"], a["Hkv"], a["d"], a["causal"],
                             a["scale"], a["dt"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(cq=None), FA_ERR_INVALID_ARG),
    (dict(ck=None), FA_ERR_INVALID_ARG),
    (dict(cq=FAKE + 2), FA_ERR_INVALID_ARG),
    (dict(uk=FAKE + 1), FA_ERR_INVALID_ARG),
    (dict(tq=0), FA_ERR_INVALID_ARG),
    (dict(tk=0), FA_ERR_INVALID_ARG),
    (dict(B=0), FA_ERR_INVALID_ARG),
    (dict(mq=0), FA_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), FA_ERR_INVALID_ARG),
    (dict(d=320), FA_ERR_UNSUPPORTED),
    (dict(q=None), FA_ERR_INVALID_ARG),
    (dict(o=FAKE + 8), FA_ERR_INVALID_ARG),
])
def test_varlen_invalid_arguments(lib, kw, code):
    assert varlen_call(lib, **kw) == code


def test_varlen_valid_arguments_reach_the_device_check(lib):
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert varlen_call(lib) in (FA_ERR_CUDA, FA_ERR_UNSUPPORTED)


def _half_ulp(ref):
    e = torch.floor(torch.log2(ref.abs().clamp_min(torch.finfo(torch.bfloat16).tiny)))
    return torch.ldexp(torch.ones_like(ref), (e - 8).to(torch.int32))


def run_varlen(oracle_mod, lens_q, lens_k, Hq, Hkv, d, causal, used_k=None, seed=0):
    import exact_attention_blackwell_fa_b200 as fa

    tq, tk = sum(lens_q), sum(lens_k)
    # draw the packed tensors with the shared generator: [1, total, H, d] -> [total, H, d]
    q, k, v = make_inputs(Shape(1, tq, tk, Hq, Hkv, d), seed=seed)
    q, k, v = q[0], k[0], v[0]
    cu_q = torch.tensor([0] + list(torch.tensor(lens_q).cumsum(0)), dtype=torch.int32)
    cu_k = torch.tensor([0] + list(torch.tensor(lens_k).cumsum(0)), dtype=torch.int32)
    uk = torch.tensor(used_k, dtype=torch.int32).cuda() if used_k is not None else None
    o, lse = fa.fa_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu_q.cuda(), cu_k.cuda(),
                              max(lens_q), max(lens_k), seqused_k=uk, causal=causal)
    torch.cuda.synchronize()
    code, detail = fa.fa_last_device_status()
    assert code == 0, f"device status {code} ({detail:#x})"
    o, lse = o.cpu().double(), lse.cpu().double()
    errs = []
    for b in range(len(lens_q)):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        k0 = int(cu_k[b])
        nk = used_k[b] if used_k is not None else lens_k[b]
        if q1 == q0:
            continue
        qs = q[q0:q1].unsqueeze(0)
        if nk == 0:  # no key: O = 0, LSE = -inf
            assert torch.all(o[q0:q1] == 0)
            assert torch.all(torch.isneginf(lse[:, q0:q1]))
            continue
        ks, vs = k[k0:k0 + nk].unsqueeze(0), v[k0:k0 + nk].unsqueeze(0)
        o_ref, lse_ref = oracle_mod.fwd(qs, ks, vs, causal=causal)
        err = (o[q0:q1] - o_ref[0]).abs()
        assert (err - (O_MAX + _half_ulp(o_ref[0]))).max().item() <= 0.0, (b, err.max().item())
        errs.append(err)
        lr = lse_ref[0]            # [Hq, Sq_b]
        lg = lse[:, q0:q1]
        fin = torch.isfinite(lr)
        assert torch.equal(torch.isfinite(lg), fin)
        if fin.any():
            assert (lg[fin] - lr[fin]).abs().max().item() <= LSE_MAX
    if errs:
        assert torch.cat([e.flatten() for e in errs]).mean().item() <= O_MEAN


CASES = [
    # lens_q, lens_k, Hq, Hkv
    ([300, 1, 128, 517], [300, 1, 128, 517], 4, 2),
    ([64, 0, 200, 256], [100, 50, 700, 256], 2, 1),      # a zero-length query sequence
    ([257, 31], [40, 900], 2, 2),                        # fewer / more keys than queries
]


@pytest.mark.gpu
@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_varlen_fwd_parity(oracle_mod, case, causal, d):
    lq, lk, Hq, Hkv = CASES[case]
    run_varlen(oracle_mod, lq, lk, Hq, Hkv, d, causal, seed=case)


@pytest.mark.gpu
@pytest.mark.parametrize("d", [128, 256])
def test_varlen_fwd_seqused_k(oracle_mod, d):
    # allocated key rows beyond seqused_k hold other data and must not take part
    run_varlen(oracle_mod, [200, 130, 90], [400, 260, 300], 4, 2, d, False, used_k=[123, 0, 300], seed=7)
    run_varlen(oracle_mod, [200, 130, 90], [400, 260, 300], 4, 2, d, True, used_k=[257, 1, 150], seed=8)


@pytest.mark.gpu
def test_varlen_matches_dense_for_equal_lengths(oracle_mod):
    """Equal lengths packed as varlen give the dense call's output bit for bit."""
    import exact_attention_blackwell_fa_b200 as fa

    B, S, H, d = 3, 384, 4, 128
    q, k, v = (t.cuda() for t in make_inputs(Shape(B, S, S, H, H, d), seed=3))
    o_d, lse_d = fa.fa_fwd(q, k, v, causal=True)
    cu = torch.arange(0, (B + 1) * S, S, dtype=torch.int32, device="cuda")
    o_v, lse_v = fa.fa_fwd_varlen(q.reshape(B * S, H, d), k.reshape(B * S, H, d), v.reshape(B * S, H, d),
                                  cu, cu, S, S, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o_v.reshape(B, S, H, d), o_d)
    assert torch.equal(lse_v.reshape(H, B, S).permute(1, 0, 2), lse_d)


# ---- backward ----------------------------------------------------------------------

GRAD_REL = 5e-2


def run_varlen_bwd(oracle_mod, lens_q, lens_k, Hq, Hkv, d, causal, used_k=None, seed=0):
    import exact_attention_blackwell_fa_b200 as fa

    tq, tk = sum(lens_q), sum(lens_k)
    q, k, v, do = make_inputs(Shape(1, tq, tk, Hq, Hkv, d), seed=seed, with_dout=True)
    q, k, v, do = q[0], k[0], v[0], do[0]
    cu_q = torch.tensor([0] + list(torch.tensor(lens_q).cumsum(0)), dtype=torch.int32)
    cu_k = torch.tensor([0] + list(torch.tensor(lens_k).cumsum(0)), dtype=torch.int32)
    uk = torch.tensor(used_k, dtype=torch.int32).cuda() if used_k is not None else None
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    mq, mk = max(lens_q), max(lens_k)
    o, lse = fa.fa_fwd_varlen(qc, kc, vc, cu_q.cuda(), cu_k.cuda(), mq, mk, seqused_k=uk, causal=causal)
    # sentinel rows: gradients of keys that take no part must stay untouched
    dk0 = torch.full_like(kc, 7.0)
    dv0 = torch.full_like(vc, 7.0)
    dq, dk, dv = fa.fa_bwd_varlen(qc, kc, vc, o, lse, doc, cu_q.cuda(), cu_k.cuda(), mq, mk, seqused_k=uk,
                                  causal=causal, dk=dk0, dv=dv0)
    torch.cuda.synchronize()
    code, detail = fa.fa_last_device_status()
    assert code == 0, f"device status {code} ({detail:#x})"
    dq, dk, dv = dq.cpu().double(), dk.cpu().double(), dv.cpu().double()
    for b in range(len(lens_q)):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        k0, k1 = int(cu_k[b]), int(cu_k[b + 1])
        nk = used_k[b] if used_k is not None else lens_k[b]
        # allocated keys past seqused_k: untouched
        assert torch.all(dk[k0 + nk:k1] == 7.0) and torch.all(dv[k0 + nk:k1] == 7.0)
        if nk == 0:
            assert torch.all(dq[q0:q1] == 0)
            continue
        if q1 == q0:  # keys without queries: zero gradients
            assert torch.all(dk[k0:k0 + nk] == 0) and torch.all(dv[k0:k0 + nk] == 0)
            continue
        sl = lambda t, a, c: t[a:c].unsqueeze(0)
        rq, rk, rv, _ = oracle_mod.bwd(sl(q, q0, q1), sl(k, k0, k0 + nk), sl(v, k0, k0 + nk), sl(do, q0, q1),
                                       causal=causal)
        scale = max(rq.abs().max().item(), rk.abs().max().item(), rv.abs().max().item())
        for name, got, ref in (("dq", dq[q0:q1], rq[0]), ("dk", dk[k0:k0 + nk], rk[0]), ("dv", dv[k0:k0 + nk], rv[0])):
            s = ref.abs().max().item() or scale
            err = (got - ref).abs().max().item()
            assert err <= GRAD_REL * s, f"seq {b} {name}: {err:.3e} > 5e-2 * {s:.3e}"


BWD_CASES = [
    ([300, 1, 128, 257], [300, 1, 128, 257], 4, 2),
    ([64, 0, 200], [100, 50, 333], 2, 1),              # a sequence with keys but no queries
    ([257, 31], [40, 300], 2, 2),
]


@pytest.mark.gpu
@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", range(len(BWD_CASES)))
def test_varlen_bwd_parity(oracle_mod, case, causal, d):
    lq, lk, Hq, Hkv = BWD_CASES[case]
    run_varlen_bwd(oracle_mod, lq, lk, Hq, Hkv, d, causal, seed=20 + case)


@pytest.mark.gpu
@pytest.mark.parametrize("d", [128, 256])
def test_varlen_bwd_seqused_k(oracle_mod, d):
    run_varlen_bwd(oracle_mod, [200, 130, 90], [400, 260, 300], 4, 2, d, False, used_k=[123, 0, 300], seed=27)
    run_varlen_bwd(oracle_mod, [200, 130, 90], [400, 260, 300], 4, 2, d, True, used_k=[257, 1, 150], seed=28)


@pytest.mark.gpu
@pytest.mark.parametrize("d", [128, 256])
def test_varlen_bwd_matches_dense_for_equal_lengths(d):
    import exact_attention_blackwell_fa_b200 as fa

    B, S, H, Hkv = 3, 384, 4, 2
    q, k, v, do = (t.cuda() for t in make_inputs(Shape(B, S, S, H, Hkv, d), seed=3, with_dout=True))
    o, lse = fa.fa_fwd(q, k, v, causal=True)
    g_d = fa.fa_bwd(q, k, v, o, lse, do, causal=True)
    cu = torch.arange(0, (B + 1) * S, S, dtype=torch.int32, device="cuda")
    pk = lambda t: t.reshape(B * S, t.shape[2], d)
    o_v, lse_v = fa.fa_fwd_varlen(pk(q), pk(k), pk(v), cu, cu, S, S, causal=True)
    g_v = fa.fa_bwd_varlen(pk(q), pk(k), pk(v), o_v, lse_v, pk(do), cu, cu, S, S, causal=True)
    torch.cuda.synchronize()
    # the dQ partial sums are reduced with floating-point atomics in a run-dependent
    # order, so dq agrees to rounding; dk and dv are accumulated in TMEM in a fixed order
    assert torch.equal(g_v[1].reshape(B, S, Hkv, d), g_d[1])
    assert torch.equal(g_v[2].reshape(B, S, Hkv, d), g_d[2])
    assert (g_v[0].reshape(B, S, H, d).float() - g_d[0].float()).abs().max().item() <= 2e-2
