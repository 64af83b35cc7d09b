"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module holds no attention arithmetic: it only draws i.i.d. normal values.
Recipe: for base seed ``s``, Q uses seed s, K s+1, V s+2 and dO s+3; each tensor is
drawn as float32 N(0, 1) with ``torch.randn`` from its own generator, multiplied by
``amp`` (0.5 for the video-diffusion shapes, 1.0 otherwise) and rounded to the
16-bit input dtype.  Layout is [batch, seq, heads, head_dim].
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Shape:
    B: int
    Sq: int
    Sk: int
    Hq: int
    Hkv: int
    d: int

    @property
    def q_shape(self):
        return (self.B, self.Sq, self.Hq, self.d)

    @property
    def kv_shape(self):
        return (self.B, self.Sk, self.Hkv, self.d)


def _draw(shape, seed, amp, dtype, device):
    g = torch.Generator(device=device).manual_seed(int(seed))
    x = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    if amp != 1.0:
        x.mul_(amp)
    return x.to(dtype)


def make_inputs(shape: Shape, seed: int = 0, dtype=torch.bfloat16, amp: float = 1.0,
                device="cpu", with_dout: bool = False):
    """Return (q, k, v) or (q, k, v, dout) drawn with the recipe above.

    ``device`` is where the values are drawn; CPU draws are the reference recipe
    used by the parity tests, CUDA draws are used only by the benchmark (which
    compares nothing against the oracle at full size).
    """
    q = _draw(shape.q_shape, seed, amp, dtype, device)
    k = _draw(shape.kv_shape, seed + 1, amp, dtype, device)
    v = _draw(shape.kv_shape, seed + 2, amp, dtype, device)
    if not with_dout:
        return q, k, v
    do = _draw(shape.q_shape, seed + 3, 1.0, dtype, device)
    return q, k, v, do


def sample_rows(B: int, H: int, S: int, n_per_head: int, seed: int = 1234,
                full_heads=()) -> torch.Tensor:
    """(n, 3) int64 list of (b, h, i) rows: every row of the heads in ``full_heads``
    (pairs (b, h)) plus ``n_per_head`` seeded random rows of every other head, always
    including the first and last row of each head."""
    g = torch.Generator().manual_seed(seed)
    out = []
    full = set(full_heads)
    for b in range(B):
        for h in range(H):
            if (b, h) in full:
                idx = torch.arange(S)
            else:
                k = max(0, min(S, n_per_head) - 2)
                idx = torch.randint(0, S, (k,), generator=g)
                idx = torch.unique(torch.cat([idx, torch.tensor([0, S - 1])]))
            bb = torch.full_like(idx, b)
            hh = torch.full_like(idx, h)
            out.append(torch.stack([bb, hh, idx], dim=1))
    return torch.cat(out, 0).to(torch.int64)
