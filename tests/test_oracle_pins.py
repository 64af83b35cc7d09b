"""Pins for the fp64 oracle, independent of the oracle's own code.

Each test fixes the oracle against something other than itself: a library
routine computing the same definition (torch's fp64 scaled_dot_product_attention
and its autograd), closed forms, invariants, finite differences and special cases
that reduce to a hand-written formula.  The definition pinned is exact attention
O = softmax(scale Q K^T [+ causal mask]) V with LSE = M + ln(l), per
"FlashAttention 4: Snellere, Geheugenefficiente Aandacht voor LLM's" (introduction,
"Slimmere Online Softmax-herwaardering").
"""
import math

import pytest
import torch
import torch.nn.functional as F

from exact_attention_blackwell_fa_b200.inputs import Shape, make_inputs

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def allowed_mask(Sq, Sk, causal):
    """Bottom-right aligned causal mask as a bool [Sq, Sk] (True = key visible)."""
    if not causal:
        return torch.ones(Sq, Sk, dtype=torch.bool)
    i = torch.arange(Sq).view(Sq, 1)
    j = torch.arange(Sk).view(1, Sk)
    return j <= i + (Sk - Sq)


def torch_reference(q, k, v, causal, scale, dout=None):
    """torch fp64 SDPA (library routine) in [B, S, H, d]; returns o, lse (+grads)."""
    qd = q.double().permute(0, 2, 1, 3).clone().requires_grad_(dout is not None)
    kd = k.double().permute(0, 2, 1, 3).clone().requires_grad_(dout is not None)
    vd = v.double().permute(0, 2, 1, 3).clone().requires_grad_(dout is not None)
    Sq, Sk = q.shape[1], k.shape[1]
    mask = allowed_mask(Sq, Sk, causal)
    o = F.scaled_dot_product_attention(qd, kd, vd, attn_mask=mask, scale=scale,
                                       enable_gqa=True)
    G = q.shape[2] // k.shape[2]
    scores = torch.matmul(qd, kd.repeat_interleave(G, dim=1).transpose(-1, -2)) * scale
    lse = torch.logsumexp(scores.masked_fill(~mask, float("-inf")), dim=-1)
    out = {"o": o.detach().permute(0, 2, 1, 3), "lse": lse.detach()}
    if dout is not None:
        (o * dout.double().permute(0, 2, 1, 3)).sum().backward()
        out["dq"] = qd.grad.permute(0, 2, 1, 3)
        out["dk"] = kd.grad.permute(0, 2, 1, 3)
        out["dv"] = vd.grad.permute(0, 2, 1, 3)
    return out


CASES = [
    # B, Sq, Sk, Hq, Hkv, d, causal
    (1, 17, 17, 2, 2, 16, False),
    (2, 33, 33, 4, 2, 8, True),
    (1, 9, 23, 3, 1, 16, True),     # Sq < Sk: bottom-right alignment
    (1, 23, 9, 2, 1, 8, True),      # Sq > Sk: the first rows see no key
    (2, 40, 31, 2, 2, 32, False),
    (1, 64, 64, 2, 2, 128, True),
    (1, 40, 50, 4, 2, 192, True),   # the library's head dims 192 and 256
    (1, 24, 24, 2, 2, 256, False),
    (1, 20, 28, 2, 1, 384, True),   # and 384, 512
    (1, 18, 18, 2, 2, 512, False),
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_forward_matches_torch_sdpa(oracle_mod, case, dtype):
    B, Sq, Sk, Hq, Hkv, d, causal = case
    q, k, v = make_inputs(Shape(B, Sq, Sk, Hq, Hkv, d), seed=3, dtype=dtype)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle_mod.fwd(q, k, v, causal=causal, scale=scale)
    ref = torch_reference(q, k, v, causal, scale)
    has_key = allowed_mask(Sq, Sk, causal).any(dim=1)            # [Sq]
    rows = has_key.view(1, Sq, 1).expand(B, Sq, Hq)
    torch.testing.assert_close(o[rows], ref["o"][rows], rtol=1e-12, atol=1e-12)
    lrows = has_key.view(1, 1, Sq).expand(B, Hq, Sq)
    torch.testing.assert_close(lse[lrows], ref["lse"][lrows], rtol=1e-12, atol=1e-12)
    # rows with no visible key: O = 0, LSE = -inf
    assert torch.all(o[~rows] == 0)
    assert torch.all(torch.isneginf(lse[~lrows]))


@pytest.mark.parametrize("case", CASES)
def test_backward_matches_torch_autograd(oracle_mod, case):
    B, Sq, Sk, Hq, Hkv, d, causal = case
    q, k, v, do = make_inputs(Shape(B, Sq, Sk, Hq, Hkv, d), seed=5, with_dout=True)
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv, D = oracle_mod.bwd(q, k, v, do, causal=causal, scale=scale)
    ref = torch_reference(q, k, v, causal, scale, dout=do)
    has_key = allowed_mask(Sq, Sk, causal).any(dim=1)
    rows = has_key.view(1, Sq, 1).expand(B, Sq, Hq)
    torch.testing.assert_close(dq[rows], ref["dq"][rows], rtol=1e-10, atol=1e-10)
    assert torch.all(dq[~rows] == 0)
    if bool(has_key.all()):
        torch.testing.assert_close(dk, ref["dk"], rtol=1e-10, atol=1e-10)
        torch.testing.assert_close(dv, ref["dv"], rtol=1e-10, atol=1e-10)
    else:
        # torch propagates NaN from the empty rows into dK/dV; compare with the empty
        # rows' dO zeroed, which removes their (zero) contribution from the reference.
        do2 = do.clone()
        do2[:, ~has_key] = 0
        q2 = q.clone()
        ref2 = torch_reference(q2, k, v, causal, scale, dout=do2)
        ok = torch.isfinite(ref2["dv"])
        torch.testing.assert_close(dv[ok], ref2["dv"][ok], rtol=1e-10, atol=1e-10)


def test_D_equals_rowsum_dO_times_O(oracle_mod):
    """D_i = sum_j P_ij dP_ij (how the oracle computes it) equals dO_i . O_i."""
    q, k, v, do = make_inputs(Shape(2, 37, 29, 4, 2, 16), seed=11, with_dout=True)
    o, _ = oracle_mod.fwd(q, k, v, causal=False)
    _, _, _, D = oracle_mod.bwd(q, k, v, do, causal=False)
    D2 = (o * do.double()).sum(-1).permute(0, 2, 1)
    torch.testing.assert_close(D, D2, rtol=1e-12, atol=1e-12)


def test_all_keys_equal_gives_mean_of_visible_values(oracle_mod):
    B, S, H, d = 1, 12, 2, 8
    q, _, v = make_inputs(Shape(B, S, S, H, H, d), seed=7)
    krow = make_inputs(Shape(1, 1, 1, H, H, d), seed=8)[1]
    k = krow.expand(B, S, H, d).contiguous()
    scale = 0.3
    for causal in (False, True):
        o, lse = oracle_mod.fwd(q, k, v, causal=causal, scale=scale)
        vd = v.double()
        for i in range(S):
            n = i + 1 if causal else S
            exp_o = vd[:, :n].mean(dim=1)                       # [B, H, d]
            torch.testing.assert_close(o[:, i], exp_o, rtol=1e-12, atol=1e-12)
            qk = (q.double()[:, i] * krow.double()[:, 0]).sum(-1)  # [B, H]
            torch.testing.assert_close(lse[:, :, i], scale * qk + math.log(n),
                                       rtol=1e-12, atol=1e-12)


def test_dominant_score_returns_that_value_row(oracle_mod):
    B, S, H, d = 1, 10, 1, 8
    q = torch.zeros(B, S, H, d, dtype=torch.bfloat16)
    k = torch.zeros(B, S, H, d, dtype=torch.bfloat16)
    q[..., 0] = 16.0
    j0 = 6
    k[:, j0, :, 0] = 16.0               # score 256 for key j0, 0 for the others
    _, _, v = make_inputs(Shape(B, S, S, H, H, d), seed=9)
    o, lse = oracle_mod.fwd(q, k, v, causal=False, scale=1.0)
    torch.testing.assert_close(o, v.double()[:, j0:j0 + 1].expand(B, S, H, d),
                               rtol=0, atol=1e-12)
    torch.testing.assert_close(lse, torch.full_like(lse, 256.0), rtol=0, atol=1e-12)


def test_causal_row0_is_v0(oracle_mod):
    q, k, v = make_inputs(Shape(2, 16, 16, 3, 3, 32), seed=13)
    o, lse = oracle_mod.fwd(q, k, v, causal=True, scale=0.25)
    torch.testing.assert_close(o[:, 0], v.double()[:, 0], rtol=0, atol=1e-13)
    qk = (q.double()[:, 0] * k.double()[:, 0]).sum(-1)
    torch.testing.assert_close(lse[:, :, 0], 0.25 * qk, rtol=1e-13, atol=1e-13)


def test_noncausal_invariant_under_joint_kv_permutation(oracle_mod):
    q, k, v = make_inputs(Shape(1, 21, 19, 2, 2, 16), seed=17)
    perm = torch.randperm(19, generator=torch.Generator().manual_seed(0))
    o1, l1 = oracle_mod.fwd(q, k, v)
    o2, l2 = oracle_mod.fwd(q, k[:, perm].contiguous(), v[:, perm].contiguous())
    torch.testing.assert_close(o1, o2, rtol=1e-12, atol=1e-12)
    torch.testing.assert_close(l1, l2, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_single_key_returns_v0_exactly(oracle_mod, dtype):
    """Sk = 1: O = V[0] bit for bit (also pins the exact 16-bit widening, including
    fp16 subnormals and large values)."""
    S, d = 9, 256
    q, k, _ = make_inputs(Shape(1, S, 1, 1, 1, d), seed=19, dtype=dtype)
    if dtype == torch.float16:
        vals = torch.tensor([6.0e-8, -6.0e-8, 3.05e-5, 6.1e-5, 1.0, -2.5, 65504.0, -65504.0])
    else:
        vals = torch.tensor([1e-38, -3e38, 3e38, 1.0, -2.5, 1e-30, 7.0, 0.0])
    v = vals.repeat(d // vals.numel()).view(1, 1, 1, d).to(dtype)
    o, lse = oracle_mod.fwd(q, k, v, causal=False)
    assert torch.equal(o, v.double().expand(1, S, 1, d))
    qk = (q.double()[:, :, 0] * k.double()[:, 0, 0]).sum(-1) / math.sqrt(d)
    torch.testing.assert_close(lse[:, 0], qk, rtol=1e-14, atol=1e-14)


def test_two_keys_one_dim_closed_form(oracle_mod):
    """d = 1, Sk = 2: O = v1 + (v0 - v1) * sigmoid(a - b), LSE = b + softplus(a - b)."""
    q = torch.tensor([0.5, -1.25, 2.0, 0.0], dtype=torch.bfloat16).view(1, 4, 1, 1)
    k = torch.tensor([1.5, -0.75], dtype=torch.bfloat16).view(1, 2, 1, 1)
    v = torch.tensor([3.0, -2.0], dtype=torch.bfloat16).view(1, 2, 1, 1)
    o, lse = oracle_mod.fwd(q, k, v, causal=False, scale=0.7)
    for i, qi in enumerate([0.5, -1.25, 2.0, 0.0]):
        a, b = 0.7 * qi * 1.5, 0.7 * qi * -0.75
        sig = 1.0 / (1.0 + math.exp(-(a - b)))
        assert abs(o[0, i, 0, 0].item() - (-2.0 + 5.0 * sig)) < 1e-14
        assert abs(lse[0, 0, i].item() - (b + math.log1p(math.exp(a - b)))) < 1e-14
    # causal with Sq = 4 > Sk = 2: rows 0, 1 see nothing, row 2 sees key 0, row 3 both
    o, lse = oracle_mod.fwd(q, k, v, causal=True, scale=0.7)
    assert o[0, 0, 0, 0].item() == 0.0 and o[0, 1, 0, 0].item() == 0.0
    assert math.isinf(lse[0, 0, 0].item()) and lse[0, 0, 0].item() < 0
    assert o[0, 2, 0, 0].item() == 3.0
    assert abs(lse[0, 0, 2].item() - 0.7 * 2.0 * 1.5) < 1e-14


def test_gqa_equals_repeated_heads(oracle_mod):
    """Hq = 4, Hkv = 2 equals Hkv = 4 with each KV head used by two consecutive query
    heads; dK/dV of the group are the sums over its query heads."""
    B, S, Hq, Hkv, d = 1, 13, 4, 2, 16
    q, k, v, do = make_inputs(Shape(B, S, S, Hq, Hkv, d), seed=23, with_dout=True)
    kr = k.repeat_interleave(2, dim=2).contiguous()
    vr = v.repeat_interleave(2, dim=2).contiguous()
    for causal in (False, True):
        o1, l1 = oracle_mod.fwd(q, k, v, causal=causal)
        o2, l2 = oracle_mod.fwd(q, kr, vr, causal=causal)
        torch.testing.assert_close(o1, o2, rtol=0, atol=0)
        torch.testing.assert_close(l1, l2, rtol=0, atol=0)
        dq1, dk1, dv1, _ = oracle_mod.bwd(q, k, v, do, causal=causal)
        dq2, dk2, dv2, _ = oracle_mod.bwd(q, kr, vr, do, causal=causal)
        torch.testing.assert_close(dq1, dq2, rtol=0, atol=0)
        torch.testing.assert_close(dk1, dk2.view(B, S, Hkv, 2, d).sum(3), rtol=1e-13, atol=1e-13)
        torch.testing.assert_close(dv1, dv2.view(B, S, Hkv, 2, d).sum(3), rtol=1e-13, atol=1e-13)


def test_backward_central_finite_differences(oracle_mod):
    """dL/dq, dL/dk, dL/dv of L = sum(dO * O) by central differences (h = 1e-6) on
    float64 inputs, with a GQA group (Hq = 2, Hkv = 1) and the causal mask."""
    g = torch.Generator().manual_seed(29)
    B, S, Hq, Hkv, d = 1, 6, 2, 1, 4
    q = torch.randn(B, S, Hq, d, generator=g, dtype=torch.float64)
    k = torch.randn(B, S, Hkv, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, S, Hkv, d, generator=g, dtype=torch.float64)
    do = torch.randn(B, S, Hq, d, generator=g, dtype=torch.float64)
    for causal in (False, True):
        dq, dk, dv, _ = oracle_mod.bwd(q, k, v, do, causal=causal, scale=0.6)

        def loss(qq, kk, vv):
            o, _ = oracle_mod.fwd(qq, kk, vv, causal=causal, scale=0.6)
            return float((o * do).sum())

        h = 1e-6
        for name, t, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = torch.zeros_like(t)
            flat = t.view(-1)
            for idx in range(flat.numel()):
                old = flat[idx].item()
                flat[idx] = old + h
                lp = loss(q, k, v)
                flat[idx] = old - h
                lm = loss(q, k, v)
                flat[idx] = old
                num.view(-1)[idx] = (lp - lm) / (2 * h)
            torch.testing.assert_close(grad, num, rtol=1e-6, atol=1e-7, msg=name)


def test_sampled_rows_match_full(oracle_mod):
    """The row-list entry points return the same values as the full computation."""
    B, Sq, Sk, Hq, Hkv, d = 2, 19, 23, 4, 2, 16
    q, k, v, do = make_inputs(Shape(B, Sq, Sk, Hq, Hkv, d), seed=31, with_dout=True)
    o, lse = oracle_mod.fwd(q, k, v, causal=True)
    dq, dk, dv, D = oracle_mod.bwd(q, k, v, do, causal=True)
    rows = torch.tensor([[0, 0, 0], [1, 3, 18], [0, 2, 7], [1, 1, 11]])
    o_r, l_r = oracle_mod.fwd(q, k, v, causal=True, rows=rows)
    kvr = torch.tensor([[0, 0, 0], [1, 1, 22], [1, 0, 5]])
    dq_r, dk_r, dv_r, D_r = oracle_mod.bwd(q, k, v, do, causal=True, qrows=rows, kvrows=kvr)
    for n, (b, h, i) in enumerate(rows.tolist()):
        assert torch.equal(o_r[n], o[b, i, h])
        assert l_r[n].item() == lse[b, h, i].item()
        assert torch.equal(dq_r[n], dq[b, i, h])
        assert D_r[n].item() == D[b, h, i].item()
    for n, (b, g, j) in enumerate(kvr.tolist()):
        torch.testing.assert_close(dk_r[n], dk[b, j, g], rtol=0, atol=0)
        torch.testing.assert_close(dv_r[n], dv[b, j, g], rtol=0, atol=0)
