"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc: a caller-owned memory pool or arena that
forbids it, a latency-critical loop that cannot afford the device-wide
synchronisation an allocation implies, an embedded host without a device allocator.
fa_bwd_noalloc gives them the backward with its scratch held in a fixed array inside
the library (32 MiB per device), so the caller passes only inputs and outputs.

This file is collected last so that a run stopping at the first failure has already
run every other test.  It must pass alone in a fresh process and after the others.
"""
import pytest
import torch

from exact_attention_blackwell_fa_b200.inputs import Shape, make_inputs

REL = 5e-2  # the backward parity tolerance: 5e-2 x the largest reference magnitude


def _problem(shape, causal, seed):
    import exact_attention_blackwell_fa_b200 as fa

    q, k, v, do = (t.cuda() for t in make_inputs(shape, seed=seed, with_dout=True))
    o, lse = fa.fa_fwd(q, k, v, causal=causal)
    return q, k, v, o, lse, do


def _assert_close(name, got, ref):
    got, ref = got.double(), ref.double()
    assert torch.isfinite(got).all(), name
    scale = max(ref.abs().max().item(), 1e-30)
    err = (got - ref).abs().max().item()
    assert err <= REL * scale, f"{name}: {err:.3e} > {REL} * {scale:.3e}"


def _oracle_close(oracle_mod, shape, causal, seed, got):
    """dQ on sampled query rows and dK / dV on sampled key rows (first and last KV
    head) against the fp64 oracle, at the backward parity tolerance."""
    from exact_attention_blackwell_fa_b200.inputs import sample_rows

    q, k, v, do = make_inputs(shape, seed=seed, with_dout=True)
    qrows = sample_rows(shape.B, shape.Hq, shape.Sq, 2, seed=seed)
    js = torch.unique(torch.tensor([0, shape.Sk // 2, shape.Sk - 1]))
    kvrows = torch.cat([torch.stack([torch.full_like(js, b), torch.full_like(js, h), js], 1)
                        for b, h in sorted({(0, 0), (shape.B - 1, shape.Hkv - 1)})])
    rq, rk, rv, _ = oracle_mod.bwd(q, k, v, do, causal=causal, qrows=qrows, kvrows=kvrows)
    dq, dk, dv = got
    gq = dq[qrows[:, 0].cuda(), qrows[:, 2].cuda(), qrows[:, 1].cuda()].cpu()
    gk = dk[kvrows[:, 0].cuda(), kvrows[:, 2].cuda(), kvrows[:, 1].cuda()].cpu()
    gv = dv[kvrows[:, 0].cuda(), kvrows[:, 2].cuda(), kvrows[:, 1].cuda()].cpu()
    for name, g, r in (("dq", gq, rq), ("dk", gk, rk), ("dv", gv, rv)):
        _assert_close(name + " vs oracle", g, r)


@pytest.mark.gpu
def test_noalloc_matches_fa_bwd_on_two_calls_in_a_row(oracle_mod):
    import exact_attention_blackwell_fa_b200 as fa
    from exact_attention_blackwell_fa_b200 import _lib

    cases = [(Shape(2, 384, 384, 4, 2, 128), True, 11),    # first call: sets up the scratch
             (Shape(1, 300, 520, 2, 2, 128), False, 12),   # second call: other sizes, reuses it
             (Shape(1, 512, 512, 2, 2, 256), True, 13),    # head_dim 256: a wider accumulator
             # just under the limit: 8 heads x 63 blocks of 128 rows = 64,512 padded rows
             (Shape(1, 8064, 8064, 8, 8, 128), False, 14)]
    for shape, causal, seed in cases:
        need = fa.fa_bwd_workspace_size(shape.B, shape.Sq, shape.Hq, shape.d)
        assert need <= _lib.FA_NOALLOC_SCRATCH_BYTES, (shape, need)
        q, k, v, o, lse, do = _problem(shape, causal, seed)
        ref = fa.fa_bwd(q, k, v, o, lse, do, causal=causal)
        got = fa.fa_bwd_noalloc(q, k, v, o, lse, do, causal=causal)
        torch.cuda.synchronize()
        code, detail = fa.fa_last_device_status()
        assert code == 0, f"device status {code} ({detail:#x})"
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            _assert_close(name, g, r)
        _oracle_close(oracle_mod, shape, causal, seed, got)
    # the near-limit problem needs all but a few KB of the array
    assert fa.fa_bwd_workspace_size(1, 8064, 8, 128) > _lib.FA_NOALLOC_SCRATCH_BYTES - 65536
    assert fa.fa_bwd_workspace_size(1, 8192, 8, 128) > _lib.FA_NOALLOC_SCRATCH_BYTES


def test_noalloc_rejects_problems_beyond_its_scratch():
    """A problem whose scratch would exceed the fixed array gets FA_ERR_SCRATCH_LIMIT
    before anything touches the device (so this runs without a GPU too)."""
    from exact_attention_blackwell_fa_b200 import _lib, build

    build.build()
    lib = _lib.load()
    assert lib.fa_bwd_workspace_size(1, 4096, 8, 128) <= _lib.FA_NOALLOC_SCRATCH_BYTES
    assert lib.fa_bwd_workspace_size(1, 8192, 16, 128) > _lib.FA_NOALLOC_SCRATCH_BYTES
    fake = 1 << 20
    code = lib.fa_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake,
                              1, 8192, 8192, 16, 16, 128, 0, 0.088, 0, None)
    assert code == _lib.FA_ERR_SCRATCH_LIMIT
    assert lib.fa_status_string(code).decode().startswith("FA_ERR_SCRATCH_LIMIT")
    # invalid arguments are still reported as such, not as a scratch problem
    code = lib.fa_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake,
                              0, 8192, 8192, 16, 16, 128, 0, 0.088, 0, None)
    assert code == _lib.FA_ERR_INVALID_ARG
