"""Host logic of bench.py that needs no GPU: the comment-insensitive source digest that
ties a recorded ncu capture to the kernels it measured, and the lookup of that record."""
import json
import os
import shutil

import bench


def test_strip_comments_keeps_code_and_literals():
    src = 'int a = 1; // note\n/* block\n comment */ asm("mov.u32 %0, 1; // kept");\nchar c = \'/\';'
    out = bench._strip_comments(src)
    assert "note" not in out and "block" not in out
    assert 'asm("mov.u32 %0, 1; // kept");' in out
    assert "char c = '/';" in out
    assert bench._strip_comments("a  =\n\n  b;") == "a = b;"


def test_digest_ignores_comments_but_not_code(tmp_path):
    src = os.path.join(bench.ROOT, "exact_attention_blackwell_fa_b200", "csrc")
    d = tmp_path / "csrc"
    shutil.copytree(src, d)
    base = bench.kernel_source_digest(str(d))
    assert base == bench.kernel_source_digest()
    f = d / "fa_fwd.cuh"
    text = f.read_text()
    f.write_text("// an added comment line\n" + text.replace("namespace fa {", "namespace fa {  /* c */", 1))
    assert bench.kernel_source_digest(str(d)) == base
    f.write_text(text.replace("kRescaleTau = 8.0f", "kRescaleTau = 7.0f", 1))
    assert bench.kernel_source_digest(str(d)) != base


def test_recorded_traffic_matches_current_sources():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for c in rec["captures"]:
        got = bench.recorded_traffic(c["kernel"], c["workload"])
        if c["source_sha256"] == bench.kernel_source_digest():
            assert got == float(c["dram_bytes_per_launch"])
        else:
            assert got is None
    assert bench.recorded_traffic("no such kernel", "no such workload") is None


def test_choose_peak_follows_the_clock_the_kernel_ran_at():
    peaks = {"bf16_tflops": 1606.3, "bf16_tflops_sustained": 1367.3, "sm_max_mhz": 1965.0,
             "clocks_under_load": {"sm_mhz_median": 1305.0}}
    p, kind, why = bench.choose_peak(peaks, {"sm_mhz": 1965.0}, 0.34)
    assert (p, kind) == (1606.3, "burst") and "1965" in why
    p, kind, _ = bench.choose_peak(peaks, {"sm_mhz": 1320.0}, 5.0)
    assert (p, kind) == (1367.3, "sustained")
    # no clock record: short regions take the burst figure, long ones the sustained
    assert bench.choose_peak(peaks, None, 0.5)[1] == "burst"
    assert bench.choose_peak(peaks, None, 4.0)[1] == "sustained"
    # fallback figures when no measured file exists
    p, kind, _ = bench.choose_peak({}, None, 0.5)
    assert p == bench.FALLBACK_PEAKS["bf16_tflops"] and kind == "burst"
