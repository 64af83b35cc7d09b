"""GPU parity at the full benchmark sizes, on outputs the oracle computes one by one.

Every configuration is run exactly as the library runs it at scale (same grids,
same persistent scheduling); the fp64 oracle then recomputes sampled rows: the
first and last query row of every head plus seeded random rows.  Shapes:

  * d=128, H=16, seqlen 1k..32k with batch = 32768 / seqlen, causal and not;
  * GQA, Hq=32, Hkv=8, seqlen 8k, batch 4;
  * d=256, 8 heads, seqlen 1k..128k with batch = max(1, 32768 / seqlen);
  * video-diffusion shapes [1, 257, 8, 128] (every row) and [1, 20480, 56, 128],
    inputs 0.5 N(0, 1);
  * backward: d=128, H=16, B=2, seqlen 4k/8k/16k, causal and not; d=256, H=8, B=1,
    seqlen 16k: dQ on sampled query rows, dK/dV on sampled key rows of the first,
    a middle and the last KV head of the first and last batch entries (the oracle
    recomputes those heads' full row statistics for them).

Tolerances are the parity tests': O max abs <= 1e-2 (+ half an output ulp), mean
<= 1e-3, LSE abs <= 1e-3; gradients max abs <= 5e-2 x the largest oracle magnitude.
"""
import pytest
import torch

from exact_attention_blackwell_fa_b200.inputs import Shape, make_inputs, sample_rows

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_MAX, GRAD_REL = 1e-2, 1e-3, 1e-3, 5e-2
ROWS_PER_HEAD = 4


def _half_ulp(ref):
    e = torch.floor(torch.log2(ref.abs().clamp_min(torch.finfo(torch.bfloat16).tiny)))
    return torch.ldexp(torch.ones_like(ref), (e - 8).to(torch.int32))


def _check_fwd(oracle_mod, shape, causal, amp=1.0, rows_per_head=ROWS_PER_HEAD, seed=0):
    import exact_attention_blackwell_fa_b200 as fa

    q, k, v = make_inputs(shape, seed=seed, amp=amp)
    o, lse = fa.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    torch.cuda.synchronize()
    code, detail = fa.fa_last_device_status()
    assert code == 0, f"device status {code} ({detail:#x})"
    rows = sample_rows(shape.B, shape.Hq, shape.Sq, rows_per_head, seed=seed + 11)
    o_ref, lse_ref = oracle_mod.fwd(q, k, v, causal=causal, rows=rows)
    b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
    got = o[b.cuda(), i.cuda(), h.cuda()].cpu().double()
    err = (got - o_ref).abs()
    assert torch.isfinite(got).all()
    excess = (err - (O_MAX + _half_ulp(o_ref))).max().item()
    assert excess <= 0.0, f"O max abs err {err.max().item():.3e}"
    assert err.mean().item() <= O_MEAN, f"O mean abs err {err.mean().item():.3e}"
    gl = lse[b.cuda(), h.cuda(), i.cuda()].cpu().double()
    fin = torch.isfinite(lse_ref)
    assert torch.equal(torch.isfinite(gl), fin)
    if fin.any():
        assert (gl[fin] - lse_ref[fin]).abs().max().item() <= LSE_MAX


SWEEP_128 = [1024, 2048, 4096, 8192, 16384, 32768]
SWEEP_256 = [1024, 2048, 4096, 8192, 16384, 32768, 65536, 98304, 131072]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S", SWEEP_128)
def test_full_fwd_d128(oracle_mod, S, causal):
    _check_fwd(oracle_mod, Shape(32768 // S, S, S, 16, 16, 128), causal)


@pytest.mark.parametrize("causal", [False, True])
def test_full_fwd_gqa(oracle_mod, causal):
    _check_fwd(oracle_mod, Shape(4, 8192, 8192, 32, 8, 128), causal)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S", SWEEP_256)
def test_full_fwd_d256(oracle_mod, S, causal):
    rows = ROWS_PER_HEAD if S <= 32768 else 2
    _check_fwd(oracle_mod, Shape(max(1, 32768 // S), S, S, 8, 8, 256), causal, rows_per_head=rows)


def test_full_fwd_video_small_every_row(oracle_mod):
    _check_fwd(oracle_mod, Shape(1, 257, 257, 8, 8, 128), False, amp=0.5, rows_per_head=257)


def test_full_fwd_video_large(oracle_mod):
    _check_fwd(oracle_mod, Shape(1, 20480, 20480, 56, 56, 128), False, amp=0.5, rows_per_head=3)


def _check_bwd(oracle_mod, shape, causal, seed=0):
    import exact_attention_blackwell_fa_b200 as fa

    q, k, v, do = make_inputs(shape, seed=seed, with_dout=True)
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.fa_fwd(qc, kc, vc, causal=causal)
    dq, dk, dv = fa.fa_bwd(qc, kc, vc, o, lse, doc, causal=causal)
    torch.cuda.synchronize()
    code, detail = fa.fa_last_device_status()
    assert code == 0, f"device status {code} ({detail:#x})"
    qrows = sample_rows(shape.B, shape.Hq, shape.Sq, 3, seed=seed + 5)
    # dK / dV: key rows of several (batch entry, KV head) pairs -- the first and the
    # last KV head, one in the middle, in the first and the last batch entry -- so that
    # a slip in mapping key blocks to heads in the persistent, L2-grouped unit order
    # shows up on some head: the first and last key of each plus two random ones
    g = torch.Generator().manual_seed(seed + 9)
    pairs = sorted({(0, 0), (shape.B - 1, shape.Hkv // 2), (shape.B - 1, shape.Hkv - 1), (0, shape.Hkv - 1)})
    kv = []
    for b_, h_ in pairs:
        js = torch.unique(torch.cat([torch.randint(0, shape.Sk, (2,), generator=g),
                                     torch.tensor([0, shape.Sk - 1])]))
        kv.append(torch.stack([torch.full_like(js, b_), torch.full_like(js, h_), js], 1))
    kvrows = torch.cat(kv)
    rq, rk, rv, _ = oracle_mod.bwd(q, k, v, do, causal=causal, qrows=qrows, kvrows=kvrows)
    b, h, i = qrows[:, 0], qrows[:, 1], qrows[:, 2]
    got_q = dq[b.cuda(), i.cuda(), h.cuda()].cpu().double()
    kb, kh, kj = kvrows[:, 0], kvrows[:, 1], kvrows[:, 2]
    got_k = dk[kb.cuda(), kj.cuda(), kh.cuda()].cpu().double()
    got_v = dv[kb.cuda(), kj.cuda(), kh.cuda()].cpu().double()
    # scale: the largest oracle magnitude among the sampled values of each tensor
    for name, got, ref in (("dq", got_q, rq), ("dk", got_k, rk), ("dv", got_v, rv)):
        assert torch.isfinite(got).all(), name
        scale = ref.abs().max().item()
        err = (got - ref).abs().max().item()
        assert err <= GRAD_REL * scale, f"{name}: {err:.3e} > 5e-2 * {scale:.3e}"


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S", [4096, 8192, 16384])
def test_full_bwd_d128(oracle_mod, S, causal):
    _check_bwd(oracle_mod, Shape(2, S, S, 16, 16, 128), causal)


def test_full_bwd_d256(oracle_mod):
    _check_bwd(oracle_mod, Shape(1, 16384, 16384, 8, 8, 256), False)


# ---- the widened rows at full size -------------------------------------------------

def _sampled_rows_check(oracle_mod, q, k, v, o, lse, causal, rows):
    """O and LSE of the given (b, h, i) rows against the oracle."""
    o_ref, lse_ref = oracle_mod.fwd(q, k, v, causal=causal, rows=rows)
    b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
    got = o[b.cuda(), i.cuda(), h.cuda()].cpu().double()
    err = (got - o_ref).abs()
    assert (err - (O_MAX + _half_ulp(o_ref))).max().item() <= 0.0, err.max().item()
    assert err.mean().item() <= O_MEAN
    gl = lse[b.cuda(), h.cuda(), i.cuda()].cpu().double()
    fin = torch.isfinite(lse_ref)
    assert torch.equal(torch.isfinite(gl), fin)
    if fin.any():
        assert (gl[fin] - lse_ref[fin]).abs().max().item() <= LSE_MAX


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_full_splitkv_decode_long_keys(oracle_mod, causal, d):
    """Decode over 128k keys: 4 sequences x 1 (and 8) queries, 32 / 4 heads."""
    import exact_attention_blackwell_fa_b200 as fa

    for Sq in (1, 8):
        shape = Shape(4, Sq, 131072, 32 if d == 128 else 16, 4 if d == 128 else 2, d)
        q, k, v = make_inputs(shape, seed=Sq)
        o, lse = fa.fa_fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=causal)
        torch.cuda.synchronize()
        assert fa.fa_last_device_status()[0] == 0
        rows = sample_rows(shape.B, shape.Hq, Sq, Sq, seed=3)
        _sampled_rows_check(oracle_mod, q, k, v, o, lse, causal, rows)


@pytest.mark.parametrize("causal", [False, True])
def test_full_pack_gqa_chunk(oracle_mod, causal):
    """A 64-query chunk against 32k keys per sequence, group of 8 (pack GQA)."""
    import exact_attention_blackwell_fa_b200 as fa

    shape = Shape(8, 64, 32768, 32, 4, 128)
    q, k, v = make_inputs(shape, seed=5)
    o, lse = fa.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    torch.cuda.synchronize()
    rows = sample_rows(shape.B, shape.Hq, shape.Sq, 2, seed=4)
    _sampled_rows_check(oracle_mod, q, k, v, o, lse, causal, rows)


@pytest.mark.parametrize("causal", [False, True])
def test_full_varlen_packed_32k_tokens(oracle_mod, causal):
    """One packed batch of 32,640 tokens (lengths 16384 .. 128), H=16, d=128: forward
    rows sampled from every sequence, and the backward's dQ on sampled rows and dK/dV
    on sampled keys of the longest and shortest sequences."""
    import exact_attention_blackwell_fa_b200 as fa

    lens = [16384, 8192, 4096, 2048, 1024, 512, 256, 128]
    H, d = 16, 128
    tot = sum(lens)
    q, k, v, do = (t[0] for t in make_inputs(Shape(1, tot, tot, H, H, d), seed=11, with_dout=True))
    cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0)), dtype=torch.int32)
    qc, kc, vc, doc, cuc = q.cuda(), k.cuda(), v.cuda(), do.cuda(), cu.cuda()
    o, lse = fa.fa_fwd_varlen(qc, kc, vc, cuc, cuc, max(lens), max(lens), causal=causal)
    dq, dk, dv = fa.fa_bwd_varlen(qc, kc, vc, o, lse, doc, cuc, cuc, max(lens), max(lens), causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    for s, L in enumerate(lens):
        a = int(cu[s])
        qs, ks, vs, dos = (t[a:a + L].unsqueeze(0) for t in (q, k, v, do))
        rows = sample_rows(1, H, L, 2, seed=s)
        b_, h_, i_ = rows[:, 0], rows[:, 1], rows[:, 2]
        o_ref, lse_ref = oracle_mod.fwd(qs, ks, vs, causal=causal, rows=rows)
        got = o[(a + i_).cuda(), h_.cuda()].cpu().double()
        err = (got - o_ref).abs()
        assert (err - (O_MAX + _half_ulp(o_ref))).max().item() <= 0.0, (L, err.max().item())
        gl = lse[h_.cuda(), (a + i_).cuda()].cpu().double()
        assert (gl - lse_ref).abs().max().item() <= LSE_MAX
        if s in (0, len(lens) - 1):
            qrows = sample_rows(1, H, L, 1, seed=s + 100)
            js = torch.unique(torch.tensor([0, L - 1, L // 2]))
            kvrows = torch.stack([torch.zeros_like(js), torch.full_like(js, H - 1), js], 1)
            rq, rk, rv, _ = oracle_mod.bwd(qs, ks, vs, dos, causal=causal, qrows=qrows, kvrows=kvrows)
            gq = dq[(a + qrows[:, 2]).cuda(), qrows[:, 1].cuda()].cpu().double()
            gk = dk[(a + js).cuda(), H - 1].cpu().double()
            gv = dv[(a + js).cuda(), H - 1].cpu().double()
            for name, g_, r_ in (("dq", gq, rq), ("dk", gk, rk), ("dv", gv, rv)):
                assert (g_ - r_).abs().max().item() <= GRAD_REL * r_.abs().max().item(), (L, name)
