#!/usr/bin/env python
"""Benchmark of the exact attention forward on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one fa_fwd call over the whole workload (default: bf16, B=2, H=32,
N=8192, d=128, causal): the tiles of Q, K, V streamed through the fused kernel
and O plus the log-sum-exp written once.  The metric is attention TFLOP/s
(4*B*H*N^2*d, halved for causal) with inputs resident in HBM; the same metric
end to end (host buffers in, host buffers out, copies included) is reported as
`e2e`.  Under torchrun every rank runs its own batch of the workload on its own
GPU (weak scaling, no collective on the data path); the job's time is the
slowest rank's.

`--impl reference` times the fp64 CPU oracle (test infrastructure, the
deliberately slow plain definition) on a bounded sample of the same workload.

`--path ring` measures the sequence-parallel forward (ring of K/V chunks,
partial results merged by log-sum-exp): under torchrun the real ring over
NCCL over the ranks of one sequence (strong scaling); on one
GPU the same schedule emulated for --ring-chunks ranks, one after another.
Each rank holds two chunks of the sequence (chunks r and 2P-1-r of 2P, the
zig-zag layout that gives every rank the same causal work).
`--path backward` measures fa_bwd (dq, dk, dv from the saved lse) on the same
workload, counting the customary 2.5x the forward's FLOPs.  `--path fp8`
measures fa_fwd_fp8 (E4M3 Q, K, V, bf16 O) on an E4M3 workload of the same
shape (default e4m3_b2h32_n8192_d128_causal) against an E4M3 cuBLAS GEMM
timed in the same run (and, beside it, the measured bf16 peak times the
nominal FP8/BF16 ratio of 2).  `--path peaks` times the bf16 and E4M3
library GEMMs alone.  `--path decode`
measures the generation step instead (fa_decode: new queries
over a resident key/value cache, HBM-bound): the metric is the cache bytes
read per second, against the measured HBM copy bandwidth.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from tiled_exact_attention_fa_b200 import accounting  # noqa: E402
from tiled_exact_attention_fa_b200 import dist as fdist  # noqa: E402
from tiled_exact_attention_fa_b200 import workloads as W  # noqa: E402

METRIC = "attention fwd TFLOPS (bf16, d=128, N=8K causal) and % of B200 dense BF16 peak"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 2**20
PROFILE_DIR = os.path.join(ROOT, "profiles")


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=W.HEADLINE.name, choices=sorted(W.BY_NAME))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--legs", default="kernel,e2e,cpu",
                    help="comma list of kernel,e2e,cpu (profiling runs use --legs kernel)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU time of the oracle sample")
    ap.add_argument("--no-clocks", action="store_true", help="do not sample nvidia-smi (profiling runs)")
    ap.add_argument("--path", default="forward", choices=["forward", "decode", "backward", "ring", "fp8", "peaks"])
    ap.add_argument("--ring-chunks", type=int, default=4,
                    help="--path ring on one GPU: sequence chunks emulated one rank after another")
    ap.add_argument("--decode-workload", default=W.DECODE_HEADLINE.name, choices=sorted(W.DECODE_BY_NAME))
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("bf16_tflops"), d.get("bf16_tflops_sustained"), d.get("hbm_gbs"), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


def kernel_digest(kind: str) -> str:
    from tiled_exact_attention_fa_b200 import build as fb
    return fb.code_digest(fb.KERNEL_SOURCES[kind])


def traffic_from_profile(w, kind: str | None = None):
    """DRAM bytes per launch from the committed ncu summary of this kernel and
    workload, or None when there is none or the kernel changed since."""
    suffix = "_bwd" if kind == "backward" else ""
    path = os.path.join(PROFILE_DIR, f"traffic_{w.name}{suffix}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if kind is None and isinstance(w, W.DecodeWorkload):
        kind = "decode_mma" if w.dtype == torch.bfloat16 else "decode"
    elif kind is None and w.dtype == torch.float8_e4m3fn:
        kind = "forward_fp8"
    elif kind is None:
        import tiled_exact_attention_fa_b200 as fa_pkg
        tile = "tile" in fa_pkg.forward_kernel_name(w.B, w.H, w.N, w.d, w.causal, w.dtype)
        kind = "forward_tile" if tile else "forward"
    if d.get("kernel_digest") != kernel_digest(kind):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "utilization.gpu",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_index: int, enabled: bool = True):
        self.gpu = gpu_index
        self.enabled = enabled
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        if not self.enabled:
            return self
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.file.flush()
        rows = []
        with open(self.file.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) != len(self.FIELDS):
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), util=float(parts[4]),
                                     reasons=[n for n, v in zip(["hw_slowdown", "hw_thermal_slowdown",
                                                                  "sw_thermal_slowdown", "sw_power_cap"],
                                                                 parts[5:]) if v.lower() == "active"]))
                except ValueError:
                    continue
        os.unlink(self.file.name)
        loaded = [r for r in rows if r["util"] >= 50] or rows
        if not loaded:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        reasons = sorted({x for r in loaded for x in r["reasons"]})
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded), "sm_max_mhz": loaded[0]["smax"],
                "reasons": reasons, "samples": len(loaded)}


def pcie_bandwidth(dev, in_bytes: int, out_bytes: int) -> dict:
    """Host<->device copy rates with pinned buffers (best of 4, CUDA events):
    each direction alone, and the time to move one step's bytes in and out
    at the same time on two streams -- the copy bound of an end-to-end step."""
    h_in = torch.empty(in_bytes, dtype=torch.uint8, pin_memory=True)
    d_in = torch.empty(in_bytes, dtype=torch.uint8, device=dev)
    h_out = torch.empty(out_bytes, dtype=torch.uint8, pin_memory=True)
    d_out = torch.empty(out_bytes, dtype=torch.uint8, device=dev)
    s = torch.cuda.current_stream(dev)
    s2 = torch.cuda.Stream(dev)

    def best_ms(body):
        best = None
        for _ in range(4):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            a.record(s)
            body()
            b.record(s)
            torch.cuda.synchronize(dev)
            ms = a.elapsed_time(b)
            best = ms if best is None else min(best, ms)
        return best

    def both():
        s2.wait_stream(s)
        d_in.copy_(h_in, non_blocking=True)
        with torch.cuda.stream(s2):
            h_out.copy_(d_out, non_blocking=True)
        s.wait_stream(s2)

    out = {"h2d_gbs": in_bytes / (best_ms(lambda: d_in.copy_(h_in, non_blocking=True)) * 1e-3) / 1e9,
           "d2h_gbs": out_bytes / (best_ms(lambda: h_out.copy_(d_out, non_blocking=True)) * 1e-3) / 1e9,
           "both_directions_ms": best_ms(both)}
    return out


def add_pcie_roofline(e2e: dict) -> None:
    """The step's copy time (both directions at once, measured) beside the
    step's time: the fraction of the end-to-end roofline reached."""
    bw = e2e["pcie"]
    bw["frac_of_copy_bound"] = bw["both_directions_ms"] / e2e["ms_per_step"]


def add_in_kernel_clock(line: dict, rec: dict, steps: int) -> None:
    """The SM clock the forward kernels themselves saw over the timed steps
    (each CTA's clock64 cycles over its global-timer nanoseconds, summed over
    CTAs): nvidia-smi samples every 200 ms, mostly between bursts, and reads
    the idle boost clock, while the kernel runs power-limited below it."""
    if not rec.get("ctas"):
        return
    c = line.setdefault("clocks", {})
    c["in_kernel_sm_mhz"] = rec["sm_mhz"]
    c["in_kernel_cycles_per_launch"] = rec["cycles_per_cta"]
    c["in_kernel_ctas_per_launch"] = rec["ctas"] / steps


def add_cycles(line: dict, ms: float) -> None:
    """Clock-neutral cost of a step beside the timed one: SM cycles per step
    (ms x the SM clock: the one the kernel measured itself where it records
    it, else the median sampled under load) and the metric scaled to the
    maximum SM clock, so runs at different (power-capped) clocks compare."""
    c = line.get("clocks") or {}
    mhz, mx = c.get("in_kernel_sm_mhz") or c.get("sm_mhz"), c.get("sm_max_mhz")
    if mhz:
        c["sm_cycles_per_step"] = ms * 1e-3 * mhz * 1e6
        c["cycles_clock"] = "in-kernel" if c.get("in_kernel_sm_mhz") else "nvidia-smi median"
        if mx and "value" in line:
            c["value_at_max_clock"] = line["value"] * mx / mhz


def sample_rows_for(w: W.Workload, seconds: float, seed: int):
    """A bounded random sample of (head, row) pairs whose oracle time is about
    `seconds` on this host; returns (rows [1, h, R], head slice, work in FLOP)."""
    import numpy as np
    import oracle
    g = torch.Generator().manual_seed(seed)
    heads = min(w.B * w.H, max(1, oracle.num_threads() // 2))
    shape = (1, heads, w.N, w.d)

    def draw():
        x = torch.randn(shape, generator=g)
        return x.to(w.dtype).float().numpy()

    q, k, v = draw(), draw(), draw()
    if w.q_mult != 1.0:
        q = q * w.q_mult
    rng = np.random.default_rng(seed)

    def run(R):
        rows = np.sort(rng.integers(0, w.N, size=(1, heads, R)), axis=-1).astype(np.int64)
        t0 = time.perf_counter()
        oracle.attention_fwd(q, k, v, w.scale, w.causal, rows=rows)
        dt = time.perf_counter() - t0
        keys = (rows + 1) if w.causal else np.full_like(rows, w.N)
        return dt, float((4.0 * w.d * keys).sum()), rows

    dt, work, _ = run(8)
    rate = work / max(dt, 1e-6)
    per_row = 4.0 * w.d * (w.N / 2 if w.causal else w.N)
    R = int(max(8, min(w.N, seconds * rate / per_row / heads)))
    return (q, k, v), heads, R, run


def cpu_leg(w: W.Workload, seconds: float):
    import oracle
    _, heads, R, run = sample_rows_for(w, seconds, seed=w.seed + 7)
    dt, work, _ = run(R)
    return {"value": work / dt / 1e12, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{heads} heads x {R} random query rows of {w.name} (fp64 oracle on host cores, "
                      f"{dt:.1f} s; work counted as 4*d per visible key)"}


def run_reference(a, w: W.Workload):
    rank, _, world = fdist.env_world()
    if rank != 0:
        return 0
    import oracle
    total_steps = a.steps + a.warmup
    per_step_s = max(0.05, min(5.0, 150.0 / max(1, total_steps)))
    _, heads, R, run = sample_rows_for(w, per_step_s, seed=w.seed + 11)
    for _ in range(a.warmup):
        run(R)
    times, works = [], []
    for _ in range(a.steps):
        dt, work, _ = run(R)
        times.append(dt)
        works.append(work)
    value = sum(works) / sum(times) / 1e12
    line = {
        "impl": "reference", "metric": FP8_METRIC if w.dtype == torch.float8_e4m3fn else METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                                        "causal": w.causal, "seed": w.seed},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"each step: {heads} heads x {R} random query rows of {w.name}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(a, w: W.Workload):
    import tiled_exact_attention_fa_b200 as fa

    rank, local_rank, world = fdist.env_world()
    if world != a.gpus:
        raise SystemExit(f"--gpus {a.gpus} but WORLD_SIZE={world}; launch N>1 with torchrun")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        fdist.init("nccl", timeout_s=300)
    legs = set(a.legs.split(","))

    # every rank runs its own batch of the workload (independent units, weak scaling)
    wr = W.Workload(w.name, w.dtype, w.B, w.H, w.N, w.d, w.causal, w.seed + 1000 * rank, w.q_mult)
    q_h, k_h, v_h = W.make_inputs(wr, pin=True)
    q, k, v = (x.to(dev, non_blocking=True) for x in (q_h, k_h, v_h))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    flops = accounting.attention_flops(w.B, w.H, w.N, w.d, w.causal)
    in_bytes = 3 * q.numel() * q.element_size()
    alg_bytes = accounting.algorithmic_bytes(w.B, w.H, w.N, w.d, q.element_size())

    def step():
        fa.forward_into(q, k, v, o, lse, scale=w.scale, causal=w.causal)

    for _ in range(a.warmup):
        step()
    fa.check_device_status()

    line = {"metric": METRIC, "unit": UNIT, "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if
            w.dtype == torch.bfloat16 else "f32", "data": "synthetic"}
    line["config"] = {
        "workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "seed": w.seed,
        "per_rank": "own seeded batch (seed + 1000*rank), no collective on the data path",
        "l2": f"inputs {in_bytes / 2**20:.0f} MiB > L2 {L2_BYTES / 2**20:.0f} MiB, no flush between steps"
        if in_bytes > L2_BYTES else "inputs smaller than L2: not flushed (not a valid headline)",
        "flop_per_step": flops}

    elapsed_ms = None
    if "kernel" in legs:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fa.clock_record(reset=True)
        with ClockSampler(local_rank, enabled=not a.no_clocks) as clocks:
            fdist.barrier(dev)
            torch.cuda.synchronize(dev)
            start.record(stream)
            for _ in range(a.steps):
                step()
            end.record(stream)
            torch.cuda.synchronize(dev)
            fdist.barrier(dev)
        fa.check_device_status()
        in_kernel = fa.clock_record(reset=True)
        elapsed_ms = fdist.max_over_ranks(start.elapsed_time(end), dev)
        ms = elapsed_ms / a.steps
        tflops_rank = flops / (ms * 1e-3) / 1e12
        peak, peak_sus, hbm, peak_kind = measured_peaks()
        line["value"] = world * tflops_rank
        line["ms_per_step"] = ms
        line["pct_of_bf16_peak"] = 100.0 * tflops_rank / peak
        line["roofline"] = {
            "bound": "tensor", "achieved": tflops_rank, "peak": peak, "unit": "TFLOP/s",
            "frac": tflops_rank / peak, "peak_kind": f"{peak_kind} dense bf16 burst (cuBLAS)",
            "frac_of_sustained": tflops_rank / peak_sus,
            "traffic": traffic_from_profile(w), "algorithmic_bytes": alg_bytes,
            "kernel": fa.forward_kernel_name(w.B, w.H, w.N, w.d, w.causal, w.dtype),
            "hbm_gbs_at_algorithmic_bytes": alg_bytes / (ms * 1e-3) / 1e9}
        line["clocks"] = clocks.summary()
        add_in_kernel_clock(line, in_kernel, a.steps)
        add_cycles(line, ms)
        line["gpu_launches"] = a.steps

    if "e2e" in legs:
        o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        l_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        fa.forward(q_h, k_h, v_h, scale=w.scale, causal=w.causal, out=(o_h, l_h))  # warm the allocator
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fdist.barrier(dev)
        torch.cuda.synchronize(dev)
        start.record(stream)
        for _ in range(a.e2e_steps):
            fa.forward(q_h, k_h, v_h, scale=w.scale, causal=w.causal, out=(o_h, l_h))
        end.record(stream)
        torch.cuda.synchronize(dev)
        fdist.barrier(dev)
        e2e_ms = fdist.max_over_ranks(start.elapsed_time(end), dev) / a.e2e_steps
        line["e2e"] = {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": e2e_ms,
                       "h2d_bytes_per_step": in_bytes,
                       "d2h_bytes_per_step": o.numel() * o.element_size() + lse.numel() * 4,
                       "api": "tiled_exact_attention_fa_b200.forward(host pinned tensors, out=host pinned) -> fa_fwd_host (C ABI; chunked, pipelined copies)",
                       "pcie": pcie_bandwidth(dev, in_bytes, o.numel() * o.element_size() + lse.numel() * 4)}
        add_pcie_roofline(line["e2e"])
        if "value" not in line:
            line["value"] = line["e2e"]["value"]

    if "cpu" in legs and rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_leg(w, a.cpu_seconds)

    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        fdist.barrier(dev)
        torch.distributed.destroy_process_group()
    return 0


FP8_METRIC = "attention fwd TFLOPS (E4M3 Q/K/V, bf16 O, d=128) and % of B200 dense FP8 peak"
FP8_DEFAULT = "e4m3_b2h32_n8192_d128_causal"


def run_fp8(a, w: W.Workload):
    """fa_fwd_fp8 on an E4M3 workload (inputs resident in HBM; e2e adds the
    host-to-device copies of Q, K, V and the copy back of O and lse)."""
    import tiled_exact_attention_fa_b200 as fa

    rank, local_rank, world = fdist.env_world()
    if world != a.gpus:
        raise SystemExit(f"--gpus {a.gpus} but WORLD_SIZE={world}; launch N>1 with torchrun")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        fdist.init("nccl", timeout_s=300)
    legs = set(a.legs.split(","))
    wr = W.Workload(w.name, w.dtype, w.B, w.H, w.N, w.d, w.causal, w.seed + 1000 * rank, w.q_mult)
    q_h, k_h, v_h = W.make_inputs(wr, pin=True)
    q, k, v = (x.to(dev, non_blocking=True) for x in (q_h, k_h, v_h))
    o = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    flops = accounting.attention_flops(w.B, w.H, w.N, w.d, w.causal)
    rows = w.B * w.H * w.N
    in_bytes = 3 * rows * w.d
    out_bytes = 2 * rows * w.d + 4 * rows
    alg_bytes = accounting.algorithmic_bytes(w.B, w.H, w.N, w.d, 1, out_elem_bytes=2)

    def step():
        fa.forward_fp8_into(q, k, v, o, lse, scale=w.scale, causal=w.causal)

    for _ in range(a.warmup):
        step()
    fa.check_device_status()
    line = {"metric": FP8_METRIC, "unit": UNIT, "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
            "data": "synthetic"}
    line["config"] = {
        "workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "seed": w.seed,
        "per_rank": "own seeded batch (seed + 1000*rank), no collective on the data path",
        "l2": f"inputs {in_bytes / 2**20:.0f} MiB > L2 {L2_BYTES / 2**20:.0f} MiB, no flush between steps"
        if in_bytes > L2_BYTES else "inputs smaller than L2: not flushed (not a valid headline)",
        "flop_per_step": flops}
    if "kernel" in legs:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fa.clock_record(reset=True)
        with ClockSampler(local_rank, enabled=not a.no_clocks) as clocks:
            fdist.barrier(dev)
            torch.cuda.synchronize(dev)
            start.record(stream)
            for _ in range(a.steps):
                step()
            end.record(stream)
            torch.cuda.synchronize(dev)
            fdist.barrier(dev)
        fa.check_device_status()
        in_kernel = fa.clock_record(reset=True)
        ms = fdist.max_over_ranks(start.elapsed_time(end), dev) / a.steps
        tflops_rank = flops / (ms * 1e-3) / 1e12
        peak, peak_sus, _, peak_kind = measured_peaks()
        line["value"] = world * tflops_rank
        line["ms_per_step"] = ms
        e4m3_peak = gemm_peak_tflops("e4m3", dev)
        line["roofline"] = {
            "bound": "tensor", "achieved": tflops_rank, "peak": e4m3_peak, "unit": "TFLOP/s",
            "frac": tflops_rank / e4m3_peak,
            "peak_kind": "measured here: cuBLAS E4M3 8192^3 (torch._scaled_mm), best of 10",
            "frac_of_nominal_ratio": tflops_rank / (2 * peak),
            "nominal_ratio_peak": f"{peak_kind} dense bf16 burst (cuBLAS) x 2, the nominal FP8/BF16 ratio",
            "frac_of_sustained": tflops_rank / (2 * peak_sus),
            "traffic": traffic_from_profile(w), "algorithmic_bytes": alg_bytes,
            "kernel": f"fa_fwd_e4m3_kernel<{str(w.causal).lower()}>",
            "hbm_gbs_at_algorithmic_bytes": alg_bytes / (ms * 1e-3) / 1e9}
        line["clocks"] = clocks.summary()
        add_in_kernel_clock(line, in_kernel, a.steps)
        add_cycles(line, ms)
        line["gpu_launches"] = a.steps
    if "e2e" in legs:
        o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        l_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)

        def e2e_step():
            # host tensors in and out: fa_fwd_fp8_host pipelines the copies with the kernel
            fa.forward_fp8_into(q_h, k_h, v_h, o_h, l_h, scale=w.scale, causal=w.causal, stream=stream)

        e2e_step()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fdist.barrier(dev)
        torch.cuda.synchronize(dev)
        start.record(stream)
        for _ in range(a.e2e_steps):
            e2e_step()
        end.record(stream)
        torch.cuda.synchronize(dev)
        fdist.barrier(dev)
        e2e_ms = fdist.max_over_ranks(start.elapsed_time(end), dev) / a.e2e_steps
        line["e2e"] = {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": e2e_ms,
                       "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out_bytes,
                       "api": "tiled_exact_attention_fa_b200.forward_fp8_into(pinned host tensors) -> "
                              "fa_fwd_fp8_host (C ABI; chunked, pipelined copies)",
                       "pcie": pcie_bandwidth(dev, in_bytes, out_bytes)}
        add_pcie_roofline(line["e2e"])
        if "value" not in line:
            line["value"] = line["e2e"]["value"]
    if "cpu" in legs and rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_leg(w, a.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        fdist.barrier(dev)
        torch.distributed.destroy_process_group()
    return 0


DECODE_METRIC = "attention decode: K/V cache bytes read per second (bf16, d=128) vs measured HBM bandwidth"
DECODE_UNIT = "GB/s"


def decode_config(w: W.DecodeWorkload) -> dict:
    return {"workload": w.name, "B": w.B, "H": w.H, "nq": w.nq, "nk": w.nk, "d": w.d, "causal": w.causal,
            "seed": w.seed}


def decode_cpu_sample(w: W.DecodeWorkload, seconds: float, seed: int):
    """Time the fp64 oracle on as many heads of the workload as fit in about
    `seconds`; returns (GB/s of cache processed, heads, elapsed s)."""
    import oracle
    g = torch.Generator().manual_seed(seed)

    def draw(n, heads):
        return torch.randn((1, heads, n, w.d), generator=g).to(w.dtype).float().numpy()

    def run(heads):
        q, k, v = draw(w.nq, heads), draw(w.nk, heads), draw(w.nk, heads)
        t0 = time.perf_counter()
        oracle.attention_decode(q, k, v, w.scale, w.causal)
        return time.perf_counter() - t0

    per_head_bytes = w.cache_bytes() / (w.B * w.H)
    dt = run(1)
    heads = int(max(1, min(w.B * w.H, seconds / max(dt, 1e-6))))
    dt = run(heads)
    return heads * per_head_bytes / dt / 1e9, heads, dt


def run_decode_reference(a, w: W.DecodeWorkload):
    rank, _, world = fdist.env_world()
    if rank != 0:
        return 0
    import oracle
    per_step_s = max(0.05, min(5.0, 150.0 / max(1, a.steps + a.warmup)))
    for _ in range(a.warmup):
        decode_cpu_sample(w, per_step_s, w.seed + 11)
    vals, times, heads = [], [], 0
    for i in range(a.steps):
        gbs, heads, dt = decode_cpu_sample(w, per_step_s, w.seed + 12 + i)
        vals.append(gbs * dt)
        times.append(dt)
    value = sum(vals) / sum(times)
    line = {"impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": DECODE_UNIT, "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": decode_config(w),
            "cpu_baseline": {"value": value, "unit": DECODE_UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"each step: {heads} heads of {w.name}"},
            "e2e": {"value": value, "unit": DECODE_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_decode(a, w: W.DecodeWorkload):
    import tiled_exact_attention_fa_b200 as fa

    rank, local_rank, world = fdist.env_world()
    if world != a.gpus:
        raise SystemExit(f"--gpus {a.gpus} but WORLD_SIZE={world}; launch N>1 with torchrun")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        fdist.init("nccl", timeout_s=300)
    legs = set(a.legs.split(","))
    wr = W.DecodeWorkload(w.name, w.dtype, w.B, w.H, w.nq, w.nk, w.d, w.causal, w.seed + 1000 * rank)
    q, k, v = W.make_decode_inputs(wr, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    ws = fa.decode_workspace(w.B, w.H, w.nq, w.nk, w.d, dev)
    stream = torch.cuda.current_stream(dev)
    esz = q.element_size()
    alg_bytes = w.cache_bytes() + 2 * q.numel() * esz + lse.numel() * 4  # K, V, Q read; O, lse written

    def step():
        fa.decode_into(q, k, v, o, lse, scale=w.scale, causal=w.causal, workspace=ws)

    for _ in range(a.warmup):
        step()
    fa.check_device_status()
    line = {"metric": DECODE_METRIC, "unit": DECODE_UNIT, "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32", "data": "synthetic"}
    line["config"] = dict(decode_config(w), per_rank="own seeded batch (seed + 1000*rank), no collective",
                          l2=f"K/V cache {w.cache_bytes() / 2**30:.1f} GiB > L2 {L2_BYTES / 2**20:.0f} MiB, no flush",
                          bytes_per_step=alg_bytes)
    if "kernel" in legs:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(local_rank, enabled=not a.no_clocks) as clocks:
            fdist.barrier(dev)
            torch.cuda.synchronize(dev)
            start.record(stream)
            for _ in range(a.steps):
                step()
            end.record(stream)
            torch.cuda.synchronize(dev)
            fdist.barrier(dev)
        fa.check_device_status()
        ms = fdist.max_over_ranks(start.elapsed_time(end), dev) / a.steps
        gbs = alg_bytes / (ms * 1e-3) / 1e9
        _, _, hbm, peak_kind = measured_peaks()
        line["value"] = world * gbs
        line["ms_per_step"] = ms
        line["roofline"] = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                            "peak_kind": f"{peak_kind} HBM copy bandwidth (a copy, reads and writes counted)",
                            "note": "the decode kernel only reads the cache; a read-only stream runs faster than "
                                    "a copy (no read/write turnaround), so frac against the copy figure can pass "
                                    "1; the nominal HBM3e bandwidth is 7700 GB/s",
                            "traffic": traffic_from_profile(w), "algorithmic_bytes": alg_bytes,
                            "kernel": f"fa_decode_mma_kernel<{w.d}>" if esz == 2 else
                            f"fa_decode_kernel<f32,{w.d},{1 if w.nq == 1 else 4}>"}
        line["clocks"] = clocks.summary()
        add_cycles(line, ms)
        line["gpu_launches"] = a.steps
    if "e2e" in legs:
        # one generation step through the public API: the new tokens' q, k, v
        # rows come from pinned host memory (k, v appended to the resident
        # cache), o and lse go back to pinned host memory
        q_h = q.cpu().pin_memory()
        kn_h = k[:, :, w.nk - w.nq:].cpu().pin_memory()
        vn_h = v[:, :, w.nk - w.nq:].cpu().pin_memory()
        o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        l_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)

        def e2e_step():
            q.copy_(q_h, non_blocking=True)
            k[:, :, w.nk - w.nq:].copy_(kn_h, non_blocking=True)
            v[:, :, w.nk - w.nq:].copy_(vn_h, non_blocking=True)
            step()
            o_h.copy_(o, non_blocking=True)
            l_h.copy_(lse, non_blocking=True)
            stream.synchronize()

        e2e_step()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fdist.barrier(dev)
        torch.cuda.synchronize(dev)
        start.record(stream)
        for _ in range(a.e2e_steps):
            e2e_step()
        end.record(stream)
        torch.cuda.synchronize(dev)
        fdist.barrier(dev)
        e2e_ms = fdist.max_over_ranks(start.elapsed_time(end), dev) / a.e2e_steps
        line["e2e"] = {"value": world * alg_bytes / (e2e_ms * 1e-3) / 1e9, "unit": DECODE_UNIT, "ms_per_step": e2e_ms,
                       "h2d_bytes_per_step": 3 * q.numel() * esz,
                       "d2h_bytes_per_step": o.numel() * esz + lse.numel() * 4,
                       "api": "new q, k, v rows host->device, tiled_exact_attention_fa_b200.decode_into -> fa_decode "
                              "(C ABI), o and lse device->host"}
        if "value" not in line:
            line["value"] = line["e2e"]["value"]
    if "cpu" in legs and rank == 0 and world == 1:
        import oracle
        gbs, heads, dt = decode_cpu_sample(w, a.cpu_seconds, w.seed + 7)
        line["cpu_baseline"] = {"value": gbs, "unit": DECODE_UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                                "sample": f"{heads} heads of {w.name} (fp64 oracle on host cores, {dt:.1f} s)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        fdist.barrier(dev)
        torch.distributed.destroy_process_group()
    return 0


BWD_METRIC = "attention bwd TFLOPS (bf16, d=128, N=8K causal; 10*B*H*N^2*d, halved for causal) and % of B200 dense BF16 peak"


def bwd_cpu_sample(w: W.Workload, seconds: float, seed: int):
    """fp64 oracle backward on whole heads of a shorter sequence (N = 512) of
    the workload's shape; returns (TFLOP/s in the metric's count, heads, s)."""
    import oracle
    n = min(w.N, 512)
    g = torch.Generator().manual_seed(seed)

    def run(heads):
        x = [torch.randn((1, heads, n, w.d), generator=g).to(w.dtype).float().numpy() for _ in range(4)]
        t0 = time.perf_counter()
        oracle.attention_bwd(*x, w.scale, w.causal)
        return time.perf_counter() - t0

    dt = run(1)
    heads = int(max(1, min(w.B * w.H, oracle.num_threads() * max(1, int(seconds / max(dt, 1e-6))))))
    dt = run(heads)
    flops = 2.5 * accounting.attention_flops(1, heads, n, w.d, w.causal)
    return flops / dt / 1e12, heads, dt, n


def bwd_algorithmic_bytes(w: W.Workload) -> int:
    """Bytes the fused backward kernel must move per launch: Q, K, V, dO read
    once, dK, dV written once, and the fp32 dQ accumulator written once (its
    reduce-adds otherwise stay in L2)."""
    t = w.B * w.H * w.N * w.d
    return 4 * t * 2 + 2 * t * 2 + t * 4


def run_backward(a, w: W.Workload):
    import tiled_exact_attention_fa_b200 as fa

    rank, local_rank, world = fdist.env_world()
    if world != a.gpus:
        raise SystemExit(f"--gpus {a.gpus} but WORLD_SIZE={world}; launch N>1 with torchrun")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        fdist.init("nccl", timeout_s=300)
    legs = set(a.legs.split(","))
    wr = W.Workload(w.name, w.dtype, w.B, w.H, w.N, w.d, w.causal, w.seed + 1000 * rank, w.q_mult)
    q_h, k_h, v_h = W.make_inputs(wr, pin=True)
    g = torch.Generator().manual_seed(wr.seed + 500)
    do_h = torch.randn(q_h.shape, generator=g).to(w.dtype).pin_memory()
    q, k, v, do = (x.to(dev, non_blocking=True) for x in (q_h, k_h, v_h, do_h))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    fa.forward_into(q, k, v, o, lse, scale=w.scale, causal=w.causal)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(int(fa.library().fa_bwd_workspace_bytes(w.B, w.H, w.N, w.d)), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    flops = 2.5 * accounting.attention_flops(w.B, w.H, w.N, w.d, w.causal)

    def step():
        fa.backward_into(q, k, v, o, lse, do, dq, dk, dv, scale=w.scale, causal=w.causal, workspace=ws)

    for _ in range(a.warmup):
        step()
    fa.check_device_status()
    line = {"metric": BWD_METRIC, "unit": UNIT, "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
                       "seed": w.seed, "pass": "backward (dq, dk, dv from the saved lse)",
                       "per_rank": "own seeded batch (seed + 1000*rank), no collective",
                       "l2": "inputs > L2, no flush", "flop_per_step": flops,
                       "mma_flop_per_step": flops}}
    if "kernel" in legs:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(local_rank, enabled=not a.no_clocks) as clocks:
            fdist.barrier(dev)
            torch.cuda.synchronize(dev)
            start.record(stream)
            for _ in range(a.steps):
                step()
            end.record(stream)
            torch.cuda.synchronize(dev)
            fdist.barrier(dev)
        fa.check_device_status()
        ms = fdist.max_over_ranks(start.elapsed_time(end), dev) / a.steps
        tf = flops / (ms * 1e-3) / 1e12
        peak, peak_sus, _, peak_kind = measured_peaks()
        line["value"] = world * tf
        line["ms_per_step"] = ms
        line["pct_of_bf16_peak"] = 100.0 * tf / peak
        line["roofline"] = {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                            "peak_kind": f"{peak_kind} dense bf16 burst (cuBLAS)", "frac_of_sustained": tf / peak_sus,
                            "traffic": traffic_from_profile(w, "backward"),
                            "algorithmic_bytes": bwd_algorithmic_bytes(w),
                            "kernel": "fa_bwd_kernel (+ fa_bwd_prep_kernel, fa_bwd_dq_convert_kernel)",
                            "note": "achieved counts 10*N^2*d (halved for causal) over the whole backward step "
                                    "(three launches); every product runs once on the tensor cores, dQ partials "
                                    "are added into an fp32 buffer by TMA reduce-adds"}
        line["clocks"] = clocks.summary()
        add_cycles(line, ms)
        line["gpu_launches"] = 3 * a.steps
    if "e2e" in legs:
        o_h = o.cpu().pin_memory()
        lse_h = lse.cpu().pin_memory()
        outs = [torch.empty(q.shape, dtype=q.dtype, pin_memory=True) for _ in range(3)]

        def e2e_step():
            for dst, src in ((q, q_h), (k, k_h), (v, v_h), (o, o_h), (lse, lse_h), (do, do_h)):
                dst.copy_(src, non_blocking=True)
            step()
            for dst, src in zip(outs, (dq, dk, dv)):
                dst.copy_(src, non_blocking=True)
            stream.synchronize()

        e2e_step()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fdist.barrier(dev)
        torch.cuda.synchronize(dev)
        start.record(stream)
        for _ in range(a.e2e_steps):
            e2e_step()
        end.record(stream)
        torch.cuda.synchronize(dev)
        fdist.barrier(dev)
        e2e_ms = fdist.max_over_ranks(start.elapsed_time(end), dev) / a.e2e_steps
        tb = q.numel() * q.element_size()
        line["e2e"] = {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": e2e_ms,
                       "h2d_bytes_per_step": 5 * tb + lse.numel() * 4, "d2h_bytes_per_step": 3 * tb,
                       "api": "host tensors -> device, tiled_exact_attention_fa_b200.backward_into -> fa_bwd, "
                              "dq, dk, dv -> host"}
        if "value" not in line:
            line["value"] = line["e2e"]["value"]
    if "cpu" in legs and rank == 0 and world == 1:
        import oracle
        tf, heads, dt, n = bwd_cpu_sample(w, a.cpu_seconds, w.seed + 7)
        line["cpu_baseline"] = {"value": tf, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                                "sample": f"{heads} heads of N={n} (d={w.d}, causal={w.causal}) through the fp64 "
                                          f"backward oracle, {dt:.1f} s; work counted as the metric counts it"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        fdist.barrier(dev)
        torch.distributed.destroy_process_group()
    return 0


RING_METRIC = "sequence-parallel attention fwd TFLOPS (bf16, d=128, N=8K causal; chunks merged by log-sum-exp)"


def ring_launches_per_rank(world: int, causal: bool) -> int:
    """Kernels one rank launches per ring step: fa_fwd per call of the
    schedule, then fa_merge per query chunk (once for the whole rows when no
    chunk-sized call was made)."""
    from tiled_exact_attention_fa_b200 import ring
    sched = ring.ring_schedule(0, world, causal)
    calls = sum(len(c) for _, _, c in sched)
    chunked = any(qp != ring.ALL for _, _, cs in sched for qp, _, _ in cs)
    return calls + (2 if chunked else 1)


def run_ring(a, w: W.Workload):
    import tiled_exact_attention_fa_b200 as fa
    from tiled_exact_attention_fa_b200 import ring

    rank, local_rank, world = fdist.env_world()
    if world != a.gpus:
        raise SystemExit(f"--gpus {a.gpus} but WORLD_SIZE={world}; launch N>1 with torchrun")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        fdist.init("nccl", timeout_s=300)
    q, k, v = (x.to(dev) for x in W.make_inputs(w))  # the whole sequence, same on every rank
    chunks = world if world > 1 else a.ring_chunks
    if w.N % (2 * chunks):
        raise SystemExit("the sequence must split into 2 * ranks equal chunks")
    ql, kl, vl = (ring.zigzag_shard(t, rank, world) for t in (q, k, v)) if world > 1 else (q, k, v)
    stream = torch.cuda.current_stream(dev)
    flops = accounting.attention_flops(w.B, w.H, w.N, w.d, w.causal)

    def step():
        if world > 1:
            return ring.ring_attention(ql, kl, vl, causal=w.causal, scale=w.scale)
        return ring.ring_attention_emulated(q, k, v, chunks, causal=w.causal, scale=w.scale)

    for _ in range(a.warmup):
        step()
    fa.check_device_status()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank, enabled=not a.no_clocks) as clocks:
        fdist.barrier(dev)
        torch.cuda.synchronize(dev)
        start.record(stream)
        for _ in range(a.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize(dev)
        fdist.barrier(dev)
    fa.check_device_status()
    ms = fdist.max_over_ranks(start.elapsed_time(end), dev) / a.steps
    tf = flops / (ms * 1e-3) / 1e12
    peak, peak_sus, _, peak_kind = measured_peaks()
    line = {"metric": RING_METRIC, "unit": UNIT, "value": tf, "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
                       "seed": w.seed, "chunks": chunks,
                       "mode": "ring over NCCL, zig-zag chunk pair per rank" if world > 1 else
                       f"{chunks} ranks (zig-zag chunk pairs) emulated one after another on one GPU",
                       "flop_per_step": flops},
            "roofline": {"bound": "tensor", "achieved": tf / world, "peak": peak, "unit": "TFLOP/s",
                         "frac": tf / world / peak, "peak_kind": f"{peak_kind} dense bf16 burst (cuBLAS)",
                         "traffic": None, "kernel": "bf16 forward kernel (chosen by size) per chunk pair + fa_merge_kernel"},
            "clocks": clocks.summary(),
            "gpu_launches": a.steps * ring_launches_per_rank(chunks, w.causal) * (1 if world > 1 else chunks)}
    add_cycles(line, ms)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        fdist.barrier(dev)
        torch.distributed.destroy_process_group()
    return 0


def gemm_peak_tflops(kind: str, dev, n: int = 8192) -> float:
    """Best-of-10 TFLOP/s of the library's dense GEMM (cuBLAS via torch) at
    M = N = K = n: kind "bf16" (torch.matmul) or "e4m3" (torch._scaled_mm,
    unit fp32 scales, bf16 out), after 3 warm-up runs."""
    g = torch.Generator(device="cpu").manual_seed(0)
    a16 = torch.randn(n, n, generator=g).to(dev, torch.bfloat16)
    b16 = torch.randn(n, n, generator=g).to(dev, torch.bfloat16)
    if kind == "bf16":
        fn = lambda: torch.matmul(a16, b16)
    else:
        a8 = a16.to(torch.float8_e4m3fn)
        b8 = b16.to(torch.float8_e4m3fn).t()  # column-major second operand, as _scaled_mm wants
        one = torch.ones((), dtype=torch.float32, device=dev)
        fn = lambda: torch._scaled_mm(a8, b8, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    for _ in range(3):
        fn()
    best = float("inf")
    for _ in range(10):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        fn()
        e.record()
        torch.cuda.synchronize()
        best = min(best, s.elapsed_time(e))
    return 2 * n ** 3 / (best * 1e-3) / 1e12


def run_peaks(a):
    """Dense GEMM throughput of the library routines on this GPU, as roofline
    denominators: cuBLAS bf16 and E4M3 (see gemm_peak_tflops)."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    with ClockSampler(0, enabled=not a.no_clocks) as clocks:
        out = {kind: gemm_peak_tflops(kind, dev) for kind in ("bf16", "e4m3")}
    line = {"metric": "dense GEMM peak (library routine)", "unit": "TFLOP/s", "value": out["e4m3"],
            "config": {"workload": "M=N=K=8192", "bf16_tflops": out["bf16"], "e4m3_tflops": out["e4m3"],
                       "e4m3_over_bf16": out["e4m3"] / out["bf16"]},
            "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)
    return 0


def main():
    a = parse()
    if a.path == "peaks":
        return run_peaks(a)
    if a.path == "ring":
        return run_ring(a, W.BY_NAME[a.workload])
    if a.path == "backward":
        return run_backward(a, W.BY_NAME[a.workload])
    if a.path == "fp8":
        w = W.BY_NAME[a.workload]
        if w.dtype != torch.float8_e4m3fn:
            w = W.BY_NAME[FP8_DEFAULT]
        if a.impl == "reference":
            return run_reference(a, w)
        return run_fp8(a, w)
    if a.path == "decode":
        wd = W.DECODE_BY_NAME[a.decode_workload]
        if a.impl == "reference":
            return run_decode_reference(a, wd)
        return run_decode(a, wd)
    w = W.BY_NAME[a.workload]
    if a.impl == "reference":
        return run_reference(a, w)
    return run_ours(a, w)


if __name__ == "__main__":
    sys.exit(main())
