"""The tiled online-softmax recurrence with a rescale threshold reaches the oracle's
result exactly (in fp64), whatever the threshold.

This is a test-only fp64 restatement of the recurrence the CUDA forward uses, in
the log2 domain: x = s * scale * log2(e); per KV tile the row reference max m is
moved to the tile's new max only when that max exceeds m by more than tau (then O
and l are multiplied by 2^(m_old - m_new)); p = 2^(x - m); l += sum p;
O += p V; finally O /= l and LSE = (m + log2 l) * ln 2.  ("FlashAttention 4:
Snellere, Geheugenefficiente Aandacht voor LLM's", section "Slimmere Online
Softmax-herwaardering": rescale only when the new maximum is significantly larger.)
The check pins the algebra of the recurrence (stale reference max shared by the
numerator and the denominator) before any kernel exists.
"""
import math

import numpy as np
import pytest
import torch

from exact_attention_blackwell_fa_b200.inputs import Shape, make_inputs

LOG2E = 1.0 / math.log(2.0)


def tiled_online_softmax(q, k, v, scale, causal, tile, tau):
    """q [Sq, d], k/v [Sk, d] float64 numpy; returns o [Sq, d], lse [Sq], rescales."""
    Sq, d = q.shape
    Sk = k.shape[0]
    o = np.zeros((Sq, d))
    lse = np.zeros(Sq)
    rescales = 0
    for i in range(Sq):
        m = -np.inf
        l = 0.0
        acc = np.zeros(d)
        for j0 in range(0, Sk, tile):
            j1 = min(Sk, j0 + tile)
            x = (k[j0:j1] @ q[i]) * scale * LOG2E
            if causal:
                cols = np.arange(j0, j1)
                x = np.where(cols <= i + (Sk - Sq), x, -np.inf)
            tmax = x.max()
            m_new = max(m, tmax)
            if m == -np.inf:
                m = m_new
            elif m_new - m > tau:
                alpha = 2.0 ** (m - m_new)
                acc *= alpha
                l *= alpha
                m = m_new
                rescales += 1
            mu = 0.0 if m == -np.inf else m
            p = np.exp2(x - mu)
            l += p.sum()
            acc += p @ v[j0:j1]
        if l > 0:
            o[i] = acc / l
            lse[i] = (m + math.log2(l)) / LOG2E
        else:
            o[i] = 0.0
            lse[i] = -np.inf
    return o, lse, rescales


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tau", [0.0, 8.0, 1e30])
@pytest.mark.parametrize("Sq,Sk", [(40, 40), (19, 45), (45, 19)])
def test_recurrence_matches_oracle(oracle_mod, causal, tau, Sq, Sk):
    d = 16
    q, k, v = make_inputs(Shape(1, Sq, Sk, 1, 1, d), seed=41, amp=2.0)
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = oracle_mod.fwd(q, k, v, causal=causal, scale=scale)
    o, lse, _ = tiled_online_softmax(q[0, :, 0].double().numpy(), k[0, :, 0].double().numpy(),
                                     v[0, :, 0].double().numpy(), scale, causal, 8, tau)
    np.testing.assert_allclose(o, o_ref[0, :, 0].numpy(), rtol=1e-12, atol=1e-12)
    fin = np.isfinite(lse_ref[0, 0].numpy())
    np.testing.assert_allclose(lse[fin], lse_ref[0, 0].numpy()[fin], rtol=1e-12, atol=1e-12)
    assert np.all(np.isneginf(lse[~fin]))


def test_threshold_cuts_rescales():
    """With a growing score trend, tau = 8 rescales far less often than tau = 0."""
    g = torch.Generator().manual_seed(3)
    d, S = 16, 256
    q = torch.randn(4, d, generator=g, dtype=torch.float64).numpy()
    k = (torch.randn(S, d, generator=g, dtype=torch.float64)
         * torch.linspace(0.2, 3.0, S, dtype=torch.float64).view(S, 1)).numpy()
    v = torch.randn(S, d, generator=g, dtype=torch.float64).numpy()
    _, _, r0 = tiled_online_softmax(q, k, v, 0.25, False, 16, 0.0)
    _, _, r8 = tiled_online_softmax(q, k, v, 0.25, False, 16, 8.0)
    assert r8 < r0
