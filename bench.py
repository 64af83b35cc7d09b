"""Benchmark: exact attention forward + backward on B200, TFLOPS and fraction of peak.

One step = the whole hot path once over one batch: fa_fwd then fa_bwd (row-sum
preprocess, dK/dV/dQ kernel, dQ conversion) on the shape
B=2, S=16384, H=16 (Hq = Hkv), d=128, non-causal, bf16, inputs N(0, 1) -- the shape
shared by the d=128 forward sweep (batch = 32768 / seqlen at 16k) and the backward
configuration (B=2, 16k).  FLOPs follow the metric's definition: forward
4*B*Hq*Sq*Sk*d (halved for causal), backward 2.5x that.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU (weak scaling, independent replicas): torchrun ... bench.py --gpus N
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = dict(B=2, S=16384, H=16, d=128, causal=False)
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
NOMINAL_BF16_TFLOPS = 2250.0


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return d, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


def _strip_comments(src):
    """C/C++ source without comments, whitespace runs collapsed (string and character
    literals kept as written), so that a comment-only edit keeps the digest."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_digest(csrc=None):
    """sha256 over the CUDA sources with comments and layout removed, to tell whether a
    recorded ncu capture still describes the kernels that run."""
    import hashlib
    csrc = csrc or os.path.join(ROOT, "exact_attention_blackwell_fa_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(csrc, name), encoding="utf-8") as f:
                h.update(name.encode() + b"\0" + _strip_comments(f.read()).encode())
    return h.hexdigest()


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` on `workload` from the ncu capture recorded in
    profiles/traffic.json, or None if there is none or the sources changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    for r in rec.get("captures", []):
        if r.get("kernel") == kernel and r.get("workload") == workload and \
                r.get("source_sha256") == kernel_source_digest():
            return float(r["dram_bytes_per_launch"])
    return None


def choose_peak(peaks, clocks, region_s):
    """The measured bf16 peak that matches how the kernel ran.

    MEASURED_PEAKS.json holds a burst figure (best of 10 short cuBLAS GEMMs, at the
    maximum SM clock) and a sustained one (a seconds-long loop under the power cap,
    at the clock median it records).  A kernel timed in a short region at close to
    the maximum clock is compared with the burst figure; one that ran for seconds, or
    whose sampled clock sat nearer the sustained loop's median, with the sustained
    figure.  Returns (peak TFLOP/s, kind, reason)."""
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sust = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    smax = float(peaks.get("sm_max_mhz", 1965.0))
    sust_mhz = float((peaks.get("clocks_under_load") or {}).get("sm_mhz_median", 0.0) or 0.0)
    mhz = clocks.get("sm_mhz") if clocks else None
    if mhz is not None and sust_mhz > 0.0:
        use_burst = abs(mhz - smax) <= abs(mhz - sust_mhz)
        why = (f"timed region {region_s:.2f} s at median {mhz:.0f} MHz SM clock, nearer the burst "
               f"clock ({smax:.0f}) than the sustained loop's median ({sust_mhz:.0f})") if use_burst else \
              (f"timed region {region_s:.2f} s at median {mhz:.0f} MHz SM clock, nearer the sustained "
               f"loop's median ({sust_mhz:.0f}) than the burst clock ({smax:.0f})")
    else:
        use_burst = region_s < 2.0
        why = f"timed region {region_s:.2f} s, {'under' if use_burst else 'over'} 2 s; no clock record"
    return (burst, "burst", why) if use_burst else (sust, "sustained", why)


def flops(B, Sq, Sk, H, d, causal):
    f = 4.0 * B * H * Sq * Sk * d
    if causal:
        f /= 2.0
    return f, 2.5 * f


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(value, device):
    """Maximum of a per-rank time over all ranks (the step time of the slowest
    replica); the value itself when not running distributed."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def oracle_cpu_baseline(budget_s=15.0):
    """Time the fp64 oracle on a bounded sample of the workload: full-length query rows
    of one head through the forward (O, LSE) and the backward dQ path.  Returns the
    oracle's rate in the metric's unit (algorithmic TFLOPS for those rows)."""
    import oracle
    from exact_attention_blackwell_fa_b200.inputs import Shape, make_inputs

    W = WORKLOAD
    # one (batch, head) slice at full sequence length stands in for the workload
    shape = Shape(1, W["S"], W["S"], 1, 1, W["d"])
    q, k, v, do = make_inputs(shape, seed=0, with_dout=True)
    nrows = 8
    done_rows = 0
    t0 = time.perf_counter()
    while True:
        rows = torch.tensor([[0, 0, (done_rows + i) % W["S"]] for i in range(nrows)])
        oracle.fwd(q, k, v, causal=W["causal"], rows=rows)
        oracle.bwd(q, k, v, do, causal=W["causal"], qrows=rows)
        done_rows += nrows
        if time.perf_counter() - t0 > budget_s:
            break
    el = time.perf_counter() - t0
    per_row = 4.0 * W["S"] * W["d"] * (1.0 + 2.5)
    return {"value": done_rows * per_row / el / 1e12, "unit": "TFLOPS",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{done_rows} full-length query rows (Sk={W['S']}, d={W['d']}) of one "
                      f"head through forward + backward-dQ, fp64, {el:.1f} s"}


# Further workloads timed in the same run (forward + backward of the pages' other
# configurations), each reported beside the headline: head_dim 256 (8 heads, 16k, the
# d=256 backward configuration) and the causal mask at head_dim 128.
EXTRA_WORKLOADS = [
    dict(B=1, S=16384, H=8, Hkv=8, d=256, causal=False),
    dict(B=2, S=16384, H=16, Hkv=16, d=128, causal=True),
    dict(B=32, S=1024, H=16, Hkv=16, d=128, causal=True),
]


def time_extra(fa, make_inputs, Shape, dev, w, steps=5, warmup=3, min_region_ms=300.0):
    """fa_fwd + fa_bwd on workload w: CUDA events around each call on the launching
    stream, L2 flushed (a 256 MiB write) before every step; mean per call.  Short
    workloads get more than `steps` timed steps, enough to fill `min_region_ms`, so
    that the clock sampler (200 ms period) sees the timed region."""
    stream = torch.cuda.current_stream(dev)
    q, k, v, do = make_inputs(Shape(w["B"], w["S"], w["S"], w["H"], w["Hkv"], w["d"]), seed=0, device=dev,
                              with_dout=True)
    o = torch.empty_like(q)
    lse = torch.empty(w["B"], w["H"], w["S"], dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_size(w["B"], w["S"], w["H"], w["d"]), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step(i, e):
        flush.fill_(i & 0xFF)
        if e:
            e[0].record(stream)
        fa.fa_fwd(q, k, v, causal=w["causal"], out=o, lse=lse, stream=stream)
        if e:
            e[1].record(stream)
        fa.fa_bwd(q, k, v, o, lse, do, causal=w["causal"], dq=dq, dk=dk, dv=dv, workspace=ws, stream=stream)
        if e:
            e[2].record(stream)

    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0.record(stream)
    for i in range(warmup):
        step(i, None)
    w1.record(stream)
    torch.cuda.synchronize(dev)
    per_step = w0.elapsed_time(w1) / max(warmup, 1)
    steps = max(steps, min(400, math.ceil(min_region_ms / max(per_step, 1e-3))))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for i in range(steps):
        step(warmup + i, ev[i])
    torch.cuda.synchronize(dev)
    code, detail = fa.fa_last_device_status(stream)
    if code != 0:
        raise RuntimeError(f"device status {code} detail {detail:#x} in extra workload {w}")
    f_fwd, f_bwd = flops(w["B"], w["S"], w["S"], w["H"], w["d"], w["causal"])
    fms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    bms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    tf, tb = f_fwd / (fms * 1e-3) / 1e12, f_bwd / (bms * 1e-3) / 1e12
    return {"workload": (f"attention fwd+bwd bf16 B={w['B']} S={w['S']} H={w['H']} Hkv={w['Hkv']} d={w['d']} "
                         f"{'causal' if w['causal'] else 'non-causal'}"),
            "steps": steps, "warmup": warmup, "l2": "flushed before every step",
            "value": (f_fwd + f_bwd) / ((fms + bms) * 1e-3) / 1e12, "unit": "TFLOPS",
            "fwd": {"ms": fms, "tflops": tf, "frac_of_2250": tf / NOMINAL_BF16_TFLOPS},
            "bwd": {"ms": bms, "tflops": tb, "frac_of_2250": tb / NOMINAL_BF16_TFLOPS},
            "gpu_launches": steps * 4}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fwd-only", action="store_true")
    # workload overrides (profiling and sweeps); the default is the benchmark workload
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--seq", type=int, default=None)
    ap.add_argument("--heads", type=int, default=None)
    ap.add_argument("--kv-heads", type=int, default=None)
    ap.add_argument("--hd", type=int, default=None)
    ap.add_argument("--causal", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the further workloads (d=256, causal) timed after the headline")
    ap.add_argument("--q-len", type=int, default=None,
                    help="query rows per sequence (default: --seq); a short one over long keys is "
                         "decode-shaped")
    ap.add_argument("--splitkv", action="store_true",
                    help="forward through fa_fwd_splitkv (slice count chosen by the library)")
    ap.add_argument("--clc", action="store_true",
                    help="forward units ordered by cluster launch control (fa_set_unit_schedule)")
    ap.add_argument("--varlen", default=None,
                    help="comma-separated sequence lengths: one packed batch of these sequences "
                         "(fa_fwd_varlen / fa_bwd_varlen) instead of the dense workload")
    args = ap.parse_args()
    if args.batch is not None:
        WORKLOAD["B"] = args.batch
    if args.seq is not None:
        WORKLOAD["S"] = args.seq
    if args.heads is not None:
        WORKLOAD["H"] = args.heads
    if args.hd is not None:
        WORKLOAD["d"] = args.hd
    if args.causal:
        WORKLOAD["causal"] = True
    WORKLOAD["Hkv"] = args.kv_heads if args.kv_heads is not None else WORKLOAD["H"]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    W = WORKLOAD
    W["Sq"] = args.q_len if args.q_len is not None else W["S"]
    lens = [int(x) for x in args.varlen.split(",")] if args.varlen else None
    if lens and (args.q_len is not None or args.splitkv):
        raise SystemExit("--varlen does not combine with --q-len / --splitkv")
    if lens:
        W["B"], W["S"] = len(lens), max(lens)
        f_fwd = sum(flops(1, L, L, W["H"], W["d"], W["causal"])[0] for L in lens)
        f_bwd = 2.5 * f_fwd
        wl = (f"attention fwd+bwd bf16 varlen packed lens={','.join(map(str, lens))} H={W['H']} "
              f"Hkv={W['Hkv']} d={W['d']} {'causal' if W['causal'] else 'non-causal'}")
    else:
        f_fwd, f_bwd = flops(W["B"], W["Sq"], W["S"], W["H"], W["d"], W["causal"])
        sq = "" if W["Sq"] == W["S"] else f" Sq={W['Sq']}"
        wl = (f"attention fwd+bwd bf16 B={W['B']} S={W['S']}{sq} H={W['H']} Hkv={W['Hkv']} d={W['d']} "
              f"{'causal' if W['causal'] else 'non-causal'}" + (" split-KV" if args.splitkv else ""))
    config = {"workload": wl,
              "B": W["B"], "seq_len": W["S"], "heads": W["H"], "kv_heads": W["Hkv"],
              "head_dim": W["d"],
              "causal": W["causal"], "global_batch": W["B"] * world,
              "parallelism": f"replicas x{world} (independent batches, no collective)",
              "l2": (f"Q, O, dO {(sum(lens) if lens else W['B'] * W['Sq']) * W['H'] * W['d'] * 2 / 2**20:.0f} MiB "
                     f"each, K, V {(sum(lens) if lens else W['B'] * W['S']) * W['Hkv'] * W['d'] * 2 / 2**20:.0f} "
                     "MiB each (L2: 126 MB)")}
    if lens:
        config["seq_lens"] = lens
    if args.clc:
        config["schedule"] = "cluster launch control"

    if args.impl == "reference":
        if rank != 0:
            return
        # The reference arm is the fp64 oracle on the host cores (no GPU code).
        steps = []
        if args.warmup:
            oracle_cpu_baseline(budget_s=1.0)
        cb = None
        for _ in range(max(1, args.steps)):
            cb = oracle_cpu_baseline(budget_s=max(2.0, 60.0 / max(1, args.steps)))
            steps.append(cb["value"])
        val = statistics.median(steps)
        print(json.dumps({
            "impl": "reference",
            "metric": "attention fwd/bwd TFLOPS at 1 B200 and fraction of 2.25 PFLOPS BF16 peak",
            "value": val, "unit": "TFLOPS", "n_gpus": 0, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "dtype": "f64",
            "data": "synthetic", "config": config,
            "cpu_baseline": {**cb, "value": val},
            "e2e": {"value": val, "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}))
        return

    import exact_attention_blackwell_fa_b200 as fa
    from exact_attention_blackwell_fa_b200.inputs import Shape, make_inputs

    if args.clc:
        fa.fa_set_unit_schedule(fa.FA_SCHED_CLC)

    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local_rank if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(dev)

    do_bwd = not args.fwd_only
    if lens:
        total = sum(lens)
        q, k, v, do = (t[0] for t in make_inputs(Shape(1, total, total, W["H"], W["Hkv"], W["d"]), seed=rank,
                                                 device=dev, with_dout=True))
        cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0)), dtype=torch.int32, device=dev)
        lse = torch.empty(W["H"], total, dtype=torch.float32, device=dev)
    else:
        shape = Shape(W["B"], W["Sq"], W["S"], W["H"], W["Hkv"], W["d"])
        q, k, v, do = make_inputs(shape, seed=rank, device=dev, with_dout=True)
        lse = torch.empty(W["B"], W["H"], W["Sq"], dtype=torch.float32, device=dev)
    o = torch.empty_like(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_size(W["B"], W["Sq"], W["H"], W["d"]), dtype=torch.uint8,
                     device=dev)
    split_ws = None
    if args.splitkv:
        from exact_attention_blackwell_fa_b200 import _lib as _fal
        need = int(_fal.load().fa_fwd_splitkv_workspace_size(W["B"], W["Sq"], W["S"], W["H"], W["Hkv"],
                                                             W["d"], 0))
        split_ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    main_bufs = dict(q=q, k=k, v=v, do=do, o=o, lse=lse, dq=dq, dk=dk, dv=dv, ws=ws)

    # the forward and backward calls through the public API, on a set of buffers
    def run_fwd(t, st):
        if lens:
            fa.fa_fwd_varlen(t["q"], t["k"], t["v"], cu, cu, W["S"], W["S"], causal=W["causal"], out=t["o"],
                             lse=t["lse"], stream=st)
        elif args.splitkv:
            fa.fa_fwd_splitkv(t["q"], t["k"], t["v"], causal=W["causal"], out=t["o"], lse=t["lse"],
                              workspace=split_ws, stream=st)
        else:
            fa.fa_fwd(t["q"], t["k"], t["v"], causal=W["causal"], out=t["o"], lse=t["lse"], stream=st)

    def run_bwd(t, st):
        if lens:
            fa.fa_bwd_varlen(t["q"], t["k"], t["v"], t["o"], t["lse"], t["do"], cu, cu, W["S"], W["S"],
                             causal=W["causal"], dq=t["dq"], dk=t["dk"], dv=t["dv"], workspace=t["ws"],
                             stream=st)
        else:
            fa.fa_bwd(t["q"], t["k"], t["v"], t["o"], t["lse"], t["do"], causal=W["causal"], dq=t["dq"],
                      dk=t["dk"], dv=t["dv"], workspace=t["ws"], stream=st)

    def step():
        run_fwd(main_bufs, stream)
        if do_bwd:
            run_bwd(main_bufs, stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    barrier()
    code, detail = fa.fa_last_device_status(stream)
    if code != 0:
        raise RuntimeError(f"device status {code} detail {detail:#x} after warm-up")

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.3)
    barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(K):
        ev[i][0].record(stream)
        run_fwd(main_bufs, stream)
        ev[i][1].record(stream)
        if do_bwd:
            run_bwd(main_bufs, stream)
        ev[i][2].record(stream)
    end.record(stream)
    barrier()
    clocks = sampler.stop()
    total_ms = max_over_ranks(start.elapsed_time(end), dev)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev) if do_bwd else 0.0
    ms_per_step = total_ms / K
    step_flops = f_fwd + (f_bwd if do_bwd else 0.0)
    value = world * step_flops / (ms_per_step * 1e-3) / 1e12
    code, detail = fa.fa_last_device_status(stream)
    if code != 0:
        raise RuntimeError(f"device status {code} detail {detail:#x} after timing")

    default_workload = not (lens or args.splitkv or args.fwd_only or any(
        x is not None for x in (args.batch, args.seq, args.heads, args.kv_heads, args.hd, args.q_len))
                            or args.causal or args.clc)
    extra = None
    if default_workload and not args.no_extra:
        extra = []
        for w in EXTRA_WORKLOADS:
            if world > 1:
                torch.distributed.barrier()
            sampler_x = ClockSampler(dev.index)
            sampler_x.start()
            r = time_extra(fa, make_inputs, Shape, dev, w)
            r["clocks"] = sampler_x.stop()
            extra.append(r)

    # end-to-end through the public API with host buffers: pinned H2D of the step's
    # inputs, the step, D2H of its outputs, all inside the timed region
    nbytes = lambda *ts: sum(t.numel() * t.element_size() for t in ts)
    h2d = nbytes(q, k, v) + (nbytes(do) if do_bwd else 0)
    d2h = nbytes(o, lse) + (nbytes(dq, dk, dv) if do_bwd else 0)
    e2e = None
    if not args.no_e2e:
        # End to end through the public API with every step's inputs copied in from
        # pinned host memory and its results (O, LSE, dQ, dK, dV) copied back, as a
        # user streaming batches would run it: copies in, compute and copies out on
        # three streams, two sets of device buffers, so step i's compute overlaps step
        # i+1's input copies and step i-1's output copies.  Timed from the first copy
        # in to the last copy out.
        hq, hk, hv, hdo = (t.cpu().pin_memory() for t in (q, k, v, do))
        sets = []
        for b in range(2):
            dbuf = {"q": torch.empty_like(q), "k": torch.empty_like(k), "v": torch.empty_like(v),
                    "do": torch.empty_like(do), "o": torch.empty_like(o), "lse": torch.empty_like(lse),
                    "dq": torch.empty_like(dq), "dk": torch.empty_like(dk), "dv": torch.empty_like(dv),
                    "ws": ws if b == 0 else torch.empty_like(ws)}
            hbuf = {n: torch.empty_like(dbuf[n], device="cpu").pin_memory()
                    for n in ("o", "lse", "dq", "dk", "dv")}
            sets.append((dbuf, hbuf))
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_done = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]
        E = max(4, K // 4)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for i in range(E):
            b = i % 2
            dbuf, hbuf = sets[b]
            if i >= 2:
                s_in.wait_event(comp_done[b])   # step i-2 no longer reads these inputs
            for n, h in (("q", hq), ("k", hk), ("v", hv)) + ((("do", hdo),) if do_bwd else ()):
                with torch.cuda.stream(s_in):
                    dbuf[n].copy_(h, non_blocking=True)
            in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            if i >= 2:
                stream.wait_event(out_done[b])  # step i-2's results have left these buffers
            run_fwd(dbuf, stream)
            if do_bwd:
                run_bwd(dbuf, stream)
            comp_done[b].record(stream)
            s_out.wait_event(comp_done[b])
            with torch.cuda.stream(s_out):
                for n in ("o", "lse") + (("dq", "dk", "dv") if do_bwd else ()):
                    hbuf[n].copy_(dbuf[n], non_blocking=True)
            out_done[b].record(s_out)
        e1.record(s_out)
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / E, dev)
        e2e = {"value": world * step_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOPS",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "pipelined": "copies in / compute / copies out on three streams, two buffer sets",
               "steps": E}

    peaks, peak_kind = load_peaks()
    # dominant kernel: the backward's dK/dV/dQ kernel when the backward runs, else the
    # forward kernel; its per-launch time is the CUDA-event time of its call
    if do_bwd and bwd_ms > fwd_ms:
        dom, dom_ms, dom_flops = "fa_bwd (dkdv + preprocess + convert)", bwd_ms, f_bwd
    else:
        dom, dom_ms, dom_flops = "fa_fwd_kernel", fwd_ms, f_fwd
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    peak, pkind, pwhy = choose_peak(peaks if peak_kind == "measured" else {}, clocks, total_ms * 1e-3)
    roof = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
            "peak_kind": f"{peak_kind} {pkind} bf16 (cuBLAS): {pwhy}", "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": recorded_traffic(dom, config["workload"])}
    if args.splitkv and not do_bwd:
        # decode-shaped: bound by reading K and V (plus Q, O, LSE) once from HBM
        alg = nbytes(q, k, v, o, lse)
        gbs = alg / (fwd_ms * 1e-3) / 1e9
        hpeak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        roof = {"bound": "hbm", "kernel": "fa_fwd_splitkv (slices + combine)", "achieved": gbs, "peak": hpeak,
                "peak_kind": f"{peak_kind} HBM copy", "unit": "GB/s", "frac": gbs / hpeak,
                "algorithmic_bytes": alg, "traffic": None}
    out = {
        "metric": "attention fwd/bwd TFLOPS at 1 B200 and fraction of 2.25 PFLOPS BF16 peak",
        "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config,
        "frac_of_2250": value / world / NOMINAL_BF16_TFLOPS,
        "fwd": {"ms": fwd_ms, "tflops": f_fwd / (fwd_ms * 1e-3) / 1e12,
                "frac_of_2250": f_fwd / (fwd_ms * 1e-3) / 1e12 / NOMINAL_BF16_TFLOPS},
        "bwd": ({"ms": bwd_ms, "tflops": f_bwd / (bwd_ms * 1e-3) / 1e12,
                 "frac_of_2250": f_bwd / (bwd_ms * 1e-3) / 1e12 / NOMINAL_BF16_TFLOPS}
                if do_bwd else None),
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": K * (1 + (3 if do_bwd else 0)),
        "clocks": clocks,
    }
    if extra is not None:
        out["extra"] = extra
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = oracle_cpu_baseline()
    if rank == 0:
        print(json.dumps(out))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
