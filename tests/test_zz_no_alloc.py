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


@pytest.mark.gpu
def test_noalloc_matches_fa_bwd_on_two_calls_in_a_row():
    import exact_attention_blackwell_fa_b200 as fa

    cases = [(Shape(2, 384, 384, 4, 2, 128), True, 11),    # first call: sets up the scratch
             (Shape(1, 300, 520, 2, 2, 128), False, 12)]   # second call: other sizes, reuses it
    for shape, causal, seed in cases:
        q, k, v, o, lse, do = _problem(shape, causal, seed)
        ref = fa.fa_bwd(q, k, v, o, lse, do, causal=causal)
        got = fa.fa_bwd_noalloc(q, k, v, o, lse, do, causal=causal)
        torch.cuda.synchronize()
        code, detail = fa.fa_last_device_status()
        assert code == 0, f"device status {code} ({detail:#x})"
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            _assert_close(name, g, r)


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
