#!/usr/bin/env python
"""Benchmark of the fused linear cross-entropy forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--parallel token|vocab] [--legs LIST]

One step is one full forward (contraction with online log-sum-exp, merge, mean)
over one batch of synthetic input already resident in HBM.  Rank 0 prints one
JSON line.  `value` and `ms_per_step` come from exactly K timed steps after W
warm-up steps.  Under torchrun (N > 1) the default `--parallel token` gives
every rank its own batch of N tokens against the same W (data-parallel, no
collective on the data path; scaling is weak) and the step time is the maximum
over ranks; `--parallel vocab` splits W's rows over the ranks instead (one
all-gather of 16 bytes per token per step; scaling is strong).

Also measured in the default run, each in its own object of the same line:
  * roofline: the forward is the contraction kernel with the merge in its
    epilogue, after a one-block kernel that clears the workspace header (the
    contraction starts early and overlaps it); the step's median duration (CUDA events on its stream)
    over a sustained window of at least --sustain-seconds, against the
    measured bf16 peaks, with the SM clock sampled during that window (median,
    and the kernel's rate binned by clock); the burst figures of the K steps
    beside it;
  * e2e: the same forward through the C ABI from pinned host buffers
    (flce_forward_host: H, y and W copied in every step, W in chunks that
    overlap the contraction; results copied back);
  * workloads: every seeded workload (tiny fp32, N=1024, N=4096 Zipf, the
    headline, the stress shape) timed the same way, each with its roofline
    fraction and the CPU oracle's time per token on the same inputs;
  * legs: the backward (dH, dW), a 4-bit quantised head (forward and dH) and
    the headline's fp32 samples (forward and backward).
`--legs none` times the headline only (for profiling captures).

``--impl reference`` times the fp64 CPU oracle instead (the reference arm).
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import re
import shutil
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_cross_entropy_bf16_b200 import synth  # noqa: E402

METRIC = "LCE fwd tokens/s & % bf16 tensor peak at N=8192 V=151936 D=4096"
# The page's fused forward at N=8192, V=151936, D=4096 took 2.105 s on an Apple
# M1 Max under MLX/Metal (D. Ineshin, "Een gefuseerde forward-kernel voor
# lineaire cross-entropy op Apple-GPU's", 2026, introduction): 8192 / 2.105 s.
PAGES_TOKENS_PER_S = 8192 / 2.105
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
# dense bf16 tensor work per SM per clock cycle on sm_100 (one 128 x 256 x 16
# tcgen05.mma in 128 cycles) and the SM count: the per-cycle peak the sampled
# clock turns into TFLOP/s
FLOP_PER_SM_CYCLE = 8192
B200_SMS = 148
L2_BYTES = 126 * 2 ** 20
FLUSH_BYTES = 256 * 2 ** 20
ALL_LEGS = ("backward", "quantized", "fp32", "workloads")
PROFILE_DIR = os.path.join(ROOT, "profiles")
# What determines the forward contraction's memory traffic: its device code
# and the host-side schedule it walks (the committed ncu traffic figure is
# used only while these files are unchanged).
KERNEL_SOURCES = ["linear_cross_entropy_bf16_b200/csrc/flce_kernels.cuh",
                  "linear_cross_entropy_bf16_b200/csrc/ptx_sm100.cuh",
                  "linear_cross_entropy_bf16_b200/csrc/flce_schedule.h"]


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def kernel_sources_sha256() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it matches the current sources."""
    path = os.path.join(PROFILE_DIR, f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_sha = re.search(r"kernel_sources_sha256:\s*([0-9a-f]{64})", text)
    m_tr = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_sha or not m_tr or m_sha.group(1) != kernel_sources_sha256():
        return None
    return float(m_tr.group(1))


def run_environment(dev) -> dict:
    """What ran: source identity, GPU, driver and library versions."""
    import torch
    env = {"kernel_sources_sha256": kernel_sources_sha256(), "gpu": torch.cuda.get_device_name(dev),
           "torch": torch.__version__, "cuda_runtime": torch.version.cuda}
    # CTA pairs on the two L2 partitions, as mapped by the first large forward
    # (the pair kernel's partition-aware order), or None if it was not taken
    import linear_cross_entropy_bf16_b200 as flce
    pm = flce.partition_map(dev)
    env["l2_partition_pairs"] = list(pm) if pm is not None else None
    try:
        h = hashlib.sha256()
        with open(os.path.abspath(__file__), "rb") as f:
            h.update(f.read())
        env["bench_sha256"] = h.hexdigest()
        out = subprocess.run(["nvidia-smi", "--query-gpu=driver_version", "--format=csv,noheader",
                              f"--id={torch.cuda.current_device()}"],
                             capture_output=True, text=True, timeout=20)
        if out.returncode == 0:
            env["driver"] = out.stdout.strip()
        g = subprocess.run(["git", "rev-parse", "HEAD"], cwd=ROOT, capture_output=True, text=True,
                           timeout=20)
        if g.returncode == 0:
            env["git"] = g.stdout.strip()
    except (OSError, subprocess.SubprocessError):
        pass
    return env


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def median(v):
    return float(np.median(np.asarray(v, dtype=np.float64))) if len(v) else float("nan")


def workload_config(w, world: int, parallel: str = "token") -> dict:
    """The workload keys of the line's `config`, the same in both arms."""
    elem = 2 if w.dtype == "bf16" else 4
    big = w.V * w.D * elem > 2 * L2_BYTES
    return {"workload": w.name, "N": w.N, "V": w.V, "D": w.D, "input_dtype": w.dtype,
            "targets": w.targets, "seed": w.seed,
            "global_batch": world * w.N if parallel == "token" else w.N,
            "parallelism": ("single GPU" if world == 1 else
                            f"dp{world}" if parallel == "token" else f"vocab-parallel over {world} GPUs"),
            "l2": (f"inputs larger than L2 (W is {w.V * w.D * elem / 1e9:.2f} GB), no flush" if big else
                   f"L2 flushed between steps (a {FLUSH_BYTES >> 20} MiB write, then a "
                   f"{FLUSH_BYTES >> 20} MiB read so that no dirty line is written back during the step)")}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of the SM clock, power and throttle reasons, with timestamps."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index: int, period_ms: int = 50):
        self.proc = None
        self.rows = []
        # the raw samples go to FLCE_BENCH_CLOCKS_DIR when set (to keep them), else a temp file
        out_dir = os.environ.get("FLCE_BENCH_CLOCKS_DIR")
        self.path = os.path.join(out_dir, f"clocks_rank{gpu_index}.csv") if out_dir \
            else os.path.join(tempfile.gettempdir(), f"flce_clocks_{os.getpid()}_{gpu_index}.csv")
        self.gpu_index = gpu_index
        self.period_ms = period_ms

    def start(self):
        if shutil.which("nvidia-smi") is None:
            return
        self.f = open(self.path, "w")
        self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                                      "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
                                     stdout=self.f, stderr=subprocess.DEVNULL)
        time.sleep(0.3)

    def stop(self):
        """Stops sampling; keeps the rows (epoch seconds, MHz, max MHz, W, active reasons)."""
        if self.proc is None:
            return
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                t = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                reasons = {self.REASONS[i] for i, v in enumerate(parts[6:10]) if v.lower() == "active"}
                self.rows.append((t, float(parts[2]), float(parts[3]), float(parts[4]), reasons))
            except ValueError:
                continue

    def summary(self, t0=None, t1=None):
        """Median SM clock of the samples drawing real power in [t0, t1], and the reasons seen."""
        rows = [r for r in self.rows if (t0 is None or r[0] >= t0) and (t1 is None or r[0] <= t1)]
        if not rows:
            return None
        loaded = [r for r in rows if r[3] > 300] or rows
        return {"sm_mhz": median([r[1] for r in loaded]), "sm_max_mhz": max(r[2] for r in rows),
                "sm_mhz_min": min(r[1] for r in rows), "samples": len(rows),
                "samples_under_load": len(loaded), "power_w_max": max(r[3] for r in rows),
                "reasons": sorted(set().union(*[r[4] for r in loaded]))}


# ----------------------------------------------------------------------------- ranks

def rank_inputs(w, rank: int):
    """Inputs of one data-parallel rank: its own tokens and targets, the shared W."""
    return synth.generate(w, token_stream=rank)


def max_over_ranks(values, world: int, device=None):
    """Element-wise maximum of a list of floats over all ranks (identity when world == 1)."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def weak_scaling_tokens_per_s(world: int, n_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes n_per_rank tokens per step."""
    return world * n_per_rank / (ms_per_step / 1e3)


def vocab_shard_bounds(V: int, world: int, rank: int):
    """Rows [a, b) of W that rank `rank` holds when W's rows are split over `world` ranks."""
    return V * rank // world, V * (rank + 1) // world


# ----------------------------------------------------------------------------- CPU oracle

def oracle_rows_timed(H, W, y, rows):
    """The oracle as it stands on the given rows, timed on the host's cores."""
    import oracle
    oracle.build()
    t0 = time.perf_counter()
    out = oracle.forward(H, W, y, rows=rows)
    return out, time.perf_counter() - t0, oracle.max_threads()


def cpu_baseline_for(w, H, W, y, rows_cap: int):
    """cpu_baseline object: the oracle on every row (workloads of at most 1024
    tokens) or on the seeded row sample the tests use (larger ones)."""
    rows = synth.sample_rows(w.N, w.N if w.N <= 1024 else rows_cap, w.seed)
    _, secs, cores = oracle_rows_timed(H, W, y, rows)
    return {"value": len(rows) / secs, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "seconds": secs, "rows": int(len(rows)), "s_per_token": secs / len(rows),
            "sample": (f"all {w.N} rows of {w.name}" if len(rows) == w.N else
                       f"{len(rows)} seeded rows of {w.name} (first and last included; full V and D "
                       f"per row)") + f", fp64, {secs:.1f} s"}


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, w, rank, world):
    """The fp64 CPU oracle as the reference implementation (rank 0 only)."""
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    H, W, y = synth.generate(w)
    cores = oracle.max_threads()
    order = np.random.default_rng([w.seed, 98]).permutation(w.N)
    per_step = cores
    pos = 0

    def step():
        nonlocal pos
        rows = order[pos % w.N: pos % w.N + per_step]
        pos += per_step
        oracle.forward(H, W, y, rows=rows)
        return len(rows)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    rows = sum(step() for _ in range(args.steps))
    dt = time.perf_counter() - t0
    value = rows / dt
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak" if args.parallel == "token" else "strong",
        "vs_baseline": value / PAGES_TOKENS_PER_S, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": workload_config(w, world, args.parallel),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{per_step} seeded rows per step of the {w.name} workload "
                                   f"({rows} rows over {args.steps} steps); fp64, logits materialised per row"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- timing helpers

class HostEvent:
    """Stand-in for torch.cuda.Event on CPU tensors (host clock)."""

    def __init__(self, **_):
        self.t = None

    def record(self, stream=None):
        self.t = time.perf_counter()

    def elapsed_time(self, other) -> float:
        return (other.t - self.t) * 1e3


def event_factory(device):
    import torch
    if device.type == "cuda":
        return lambda: torch.cuda.Event(enable_timing=True)
    return HostEvent


def sync(device):
    import torch
    if device.type == "cuda":
        torch.cuda.synchronize(device)


class ForwardTimer:
    """One forward step: flce_forward, two launches (a one-block header clear, and
    the contraction with the merge in its epilogue, which starts early and overlaps
    it), between two CUDA events on the launching stream."""

    def __init__(self, flce, H, W, y, dev, stream):
        import torch
        N, V, D = H.shape[0], W.shape[0], H.shape[1]
        self.flce, self.H, self.W, self.y, self.stream, self.dev = flce, H, W, y, stream, dev
        self.ws = torch.empty(flce.workspace_size(N, V, D, H.dtype), dtype=torch.uint8, device=dev)
        self.out = {"loss": torch.empty(N, device=dev), "lse": torch.empty(N, device=dev),
                    "target_logit": torch.empty(N, device=dev), "mean": torch.empty((), device=dev)}
        self.lse, self.mean = self.out["lse"], self.out["mean"]

    def run(self, steps: int, flush=None):
        """Times `steps` steps; returns the per-step times (ms) and the total ms from the
        first step's start to the last step's end.  `flush`: a (write, read) pair of
        buffers larger than L2, written and then read between steps."""
        import torch
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        with torch.cuda.stream(self.stream):
            for k in range(steps):
                if flush is not None:
                    flush[0].zero_()
                    flush[1].sum(dtype=torch.float32)
                ev[k][0].record(self.stream)
                self.flce.forward(self.H, self.W, self.y, out=self.out, workspace=self.ws,
                                  stream=self.stream)
                ev[k][1].record(self.stream)
        torch.cuda.synchronize(self.dev)
        step = [ev[k][0].elapsed_time(ev[k][1]) for k in range(steps)]
        return step, ev[0][0].elapsed_time(ev[steps - 1][1])

    def check(self, what):
        st = self.flce.check(self.ws, self.stream)
        if st != self.flce.OK:
            raise self.flce.FlceError(st, what)


def roofline_numbers(flops: float, kernel_ms: float, peaks: dict) -> dict:
    tf = flops / (kernel_ms * 1e-3) / 1e12
    return {"tflops": tf, "frac_of_bf16_peak": tf / peaks["bf16_tflops"],
            "frac_of_sustained_peak": tf / peaks["bf16_tflops_sustained"]}


def sustained_window(timer: ForwardTimer, seconds: float, chunk_steps: int = 20):
    """Back-to-back steps for at least `seconds`, in chunks of `chunk_steps` whose host
    time spans are matched to the clock samples.  Returns the chunks (t0, t1, step ms
    list)."""
    chunks = []
    t_end = time.time() + seconds
    while time.time() < t_end or len(chunks) < 3:
        sync(timer.dev)
        t0 = time.time()
        step, _ = timer.run(chunk_steps)
        chunks.append((t0, time.time(), step))
    return chunks


def sustained_summary(chunks, flops: float, N: int, peaks: dict, sampler: ClockSampler) -> dict:
    """Medians of the sustained window's steps (the contraction kernel is all but a
    microsecond of a step), their rate against the peaks, and by clock."""
    kern = [v for c in chunks for v in c[2]]
    km = median(kern)
    res = {"seconds": chunks[-1][1] - chunks[0][0], "steps": len(kern),
           "ms_per_step_median": km, "tokens_per_s_median_step": N / (km * 1e-3),
           "kernel_ms_median": km, "kernel_ms_mean": float(np.mean(kern)),
           "kernel_ms_p10": float(np.percentile(kern, 10)), "kernel_ms_p90": float(np.percentile(kern, 90)),
           **roofline_numbers(flops, km, peaks)}
    clocks = sampler.summary(chunks[0][0], chunks[-1][1])
    res["clocks"] = clocks
    if clocks:
        per_cycle = B200_SMS * FLOP_PER_SM_CYCLE * clocks["sm_mhz"] * 1e6 / 1e12
        res["tflops_per_mhz"] = res["tflops"] / clocks["sm_mhz"]
        res["frac_of_per_cycle_peak_at_median_clock"] = res["tflops"] / per_cycle
        # per chunk: the clock samples that fall inside its host time span
        bins = {}
        for t0, t1, kc in chunks:
            mhz = [r[1] for r in sampler.rows if t0 <= r[0] <= t1 and r[3] > 300]
            if not mhz:
                continue
            b = int(round(median(mhz) / 50.0) * 50)
            bins.setdefault(b, []).extend(kc)
        res["by_clock"] = [
            {"sm_mhz_bin": b, "steps": len(v), "kernel_ms_median": median(v),
             "tflops": flops / (median(v) * 1e-3) / 1e12,
             "tflops_per_mhz": flops / (median(v) * 1e-3) / 1e12 / b}
            for b, v in sorted(bins.items())]
    return res


# ----------------------------------------------------------------------------- our arm

def to_device_tensors(Hn, Wn, yn, dev, pin=False):
    import torch

    def host_tensor(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return t.view(torch.bfloat16) if a.dtype == np.uint16 else t

    H_h, W_h, y_h = host_tensor(Hn), host_tensor(Wn), torch.from_numpy(yn)
    if pin:
        H_h, W_h, y_h = H_h.pin_memory(), W_h.pin_memory(), y_h.pin_memory()
    return (H_h, W_h, y_h), (H_h.to(dev), W_h.to(dev), y_h.to(dev))


def run_ours(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import linear_cross_entropy_bf16_b200 as flce
    from linear_cross_entropy_bf16_b200 import build as lib_build

    if rank == 0:
        lib_build.build()
    if world > 1:
        dist.barrier()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    flce.load_library()
    legs = set(args.legs)
    peaks, peak_kind = measured_peaks()

    # inputs: W is the shared projection; each rank has its own tokens and targets
    t0 = time.perf_counter()
    Hn, Wn, yn = rank_inputs(w, rank)
    log(f"[rank {rank}] generated inputs in {time.perf_counter() - t0:.1f} s")
    (H_h, W_h, y_h), (H, W, y) = to_device_tensors(Hn, Wn, yn, dev, pin=True)
    N, V, D = w.N, w.V, w.D
    flops = w.flops
    stream = torch.cuda.Stream(dev)
    fwd = ForwardTimer(flce, H, W, y, dev, stream)

    for _ in range(max(3, args.warmup)):
        fwd.run(1)
    fwd.check("warm-up")

    # ---- timed region: exactly K steps, per-kernel events on the launching stream
    K = args.steps
    sampler = ClockSampler(local_rank)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_timed = time.time()
    part_ms, total_ms = fwd.run(K)
    t_timed_end = time.time()
    if world > 1:
        dist.barrier()
    fwd.check("timed region")
    mean_loss = float(fwd.mean.item())

    # ---- sustained window: the same steps back to back for >= sustain_seconds
    chunks = sustained_window(fwd, args.sustain_seconds) if args.sustain_seconds > 0 else []
    if world > 1:
        dist.barrier()
    sampler.stop()
    fwd.check("sustained window")
    sustained = sustained_summary(chunks, flops, N, peaks, sampler) if chunks else None

    # ---- end to end through the public API from pinned host memory
    e2e = time_e2e(flce, fwd, H_h, W_h, y_h, w, dev, stream, args, world, mean_loss)

    # ---- max over ranks
    total_ms, part_med, part_mean = max_over_ranks(
        [total_ms, median(part_ms), float(np.mean(part_ms))], world, device=dev)
    sus_med = max_over_ranks([sustained["kernel_ms_median"] if sustained else part_med], world, device=dev)[0]

    # the optional legs take their own max over ranks: every rank runs them
    extra = {}
    if "backward" in legs and w.dtype == "bf16":
        extra["backward"] = time_backward(flce, H, W, y, fwd.lse, N, V, D, dev, stream, args, peaks, world,
                                          local_rank)
    if "quantized" in legs and w.dtype == "bf16":
        bits, gs = (int(v) for v in args.quantized.split(","))
        extra["quantized"] = time_quantized(flce, H, Wn, y, N, V, D, bits, gs, dev, stream, args, peaks,
                                            world)
    if "fp32" in legs and w.dtype == "bf16":
        extra["fp32"] = time_fp32(flce, w, rank, y, dev, stream, args, peaks, world)
    del fwd
    workloads = None
    host_inputs = {w.name: (Hn, Wn, yn)}
    if "workloads" in legs and world == 1:
        workloads = {}
        flush = (torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev),
                 torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev))
        for name, wl in synth.WORKLOADS.items():
            if name == w.name:
                continue
            workloads[name], host_inputs[name] = time_workload(flce, wl, dev, stream, args, peaks, flush)
        del flush

    if rank != 0:
        return 0

    ms_step = total_ms / K
    tokens_per_s = weak_scaling_tokens_per_s(world, N, ms_step)
    p = flce.plan(N, V, D, H.dtype)
    kernel = "flce_tc2_kernel" if p["ctas_per_unit"] == 2 else "flce_tc_kernel"
    achieved = flops / (sus_med * 1e-3) / 1e12
    line = {
        "metric": METRIC,
        "value": tokens_per_s,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": max(3, args.warmup),
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": tokens_per_s / PAGES_TOKENS_PER_S,
        "vs_baseline_note": "divides by the page's fused forward on an Apple M1 Max (8192 tokens / 2.105 s): context, other hardware",
        "dtype": "bf16" if w.dtype == "bf16" else "fp32",
        "data": "synthetic (seeded numpy: H~N(0,1), W~N(0,1/D), targets per workload)",
        "config": workload_config(w, world, "token"),
        "roofline": {"bound": "tensor", "kernel": kernel,
                     "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"],
                     "peak_kind": f"{peak_kind} burst bf16 (MEASURED_PEAKS.json bf16_tflops)",
                     "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                     "kernel_ms": sus_med,
                     "kernel_ms_from": (f"median over the sustained window ({sustained['steps']} steps, "
                                        f"{sustained['seconds']:.1f} s)") if sustained else
                                       f"median over the {K} timed steps",
                     "burst": {"kernel_ms_mean": part_mean, "kernel_ms_median": part_med,
                               "frac_from_mean": flops / (part_mean * 1e-3) / 1e12 / peaks["bf16_tflops"],
                               "window_s": (t_timed_end - t_timed)},
                     "flops_per_launch": flops,
                     "traffic": profiled_traffic(w.name, kernel)},
        "sustained": sustained,
        "e2e": e2e["e2e"],
        "e2e_resident_head": e2e["resident"],
        "gpu_launches": 2 * K,  # per step: the header clear and the contraction
        "kernel_ms_stats": {"median": median(part_ms), "min": float(np.min(part_ms)),
                            "max": float(np.max(part_ms)), "mean": float(np.mean(part_ms))},
        "env": run_environment(dev),
        "clocks": sampler.summary(),
        "mean_loss": mean_loss,
    }
    line.update(extra)
    if workloads is not None:
        workloads[w.name] = headline_entry(w, ms_step, part_med, sus_med, peaks, kernel)
    if world == 1 and not args.no_cpu_baseline:
        head = cpu_baseline_for(w, Hn, Wn, yn, args.cpu_rows)
        line["cpu_baseline"] = head
        if workloads is not None:
            for name, (h_, w_, y_) in host_inputs.items():
                workloads[name]["cpu_baseline"] = head if name == w.name else \
                    cpu_baseline_for(synth.WORKLOADS[name], h_, w_, y_, args.cpu_rows)
                workloads[name]["vs_cpu_oracle"] = workloads[name]["tokens_per_s"] / \
                    workloads[name]["cpu_baseline"]["value"]
    if workloads is not None:
        line["workloads"] = {n: workloads[n] for n in synth.WORKLOADS if n in workloads}
    if world == 1 and args.context:
        line["context"] = torch_materialised(H, W, y, dev)
    print(json.dumps(line), flush=True)
    return 0


def headline_entry(w, ms_step, part_med, sus_med, peaks, kernel):
    return {"N": w.N, "V": w.V, "D": w.D, "input_dtype": w.dtype, "targets": w.targets,
            "ms_per_step": ms_step, "tokens_per_s": w.N / (ms_step * 1e-3), "kernel": kernel,
            "kernel_ms": sus_med, "kernel_ms_burst_median": part_med,
            **roofline_numbers(w.flops, sus_med, peaks),
            "l2": "inputs larger than L2, no flush",
            "what": "the headline: the K timed steps for the step time, the sustained window for the kernel"}


def time_workload(flce, w, dev, stream, args, peaks, flush):
    """One seeded workload at full size: median step and contraction-kernel times over
    max(steps, 20) steps after 3 warm-up steps, the L2 flushed between steps when the
    inputs fit in it."""
    import torch
    Hn, Wn, yn = synth.generate(w)
    _, (H, W, y) = to_device_tensors(Hn, Wn, yn, dev)
    t = ForwardTimer(flce, H, W, y, dev, stream)
    elem = 2 if w.dtype == "bf16" else 4
    needs_flush = w.V * w.D * elem <= 2 * L2_BYTES
    for _ in range(3):
        t.run(1, flush if needs_flush else None)
    steps = max(20, args.steps)
    kern, _ = t.run(steps, flush if needs_flush else None)
    t.check(w.name)
    km = sm = median(kern)
    p = flce.plan(w.N, w.V, w.D, H.dtype)
    res = {"N": w.N, "V": w.V, "D": w.D, "input_dtype": w.dtype, "targets": w.targets,
           "steps": steps, "ms_per_step": sm, "tokens_per_s": w.N / (sm * 1e-3),
           "kernel": "flce_tc2_kernel" if p["ctas_per_unit"] == 2 else "flce_tc_kernel",
           "kernel_ms": km, "kernel_ms_min": float(np.min(kern)), **roofline_numbers(w.flops, km, peaks),
           "l2": "flushed between steps" if needs_flush else "inputs larger than L2, no flush",
           "mean_loss": float(t.mean.item())}
    # DRAM bytes per launch from the committed ncu summary of this kernel and workload
    # (null when there is none, or when the kernel's sources changed since it was taken)
    res["traffic"] = profiled_traffic(w.name, res["kernel"])
    if w.dtype == "fp32":
        Dp = (w.D + 63) // 64 * 64
        tensor = 2 * w.N * w.V * 3 * Dp
        res["tensor_tflops"] = tensor / (km * 1e-3) / 1e12
        res["tensor_frac_of_bf16_peak"] = res["tensor_tflops"] / peaks["bf16_tflops"]
        res["note"] = ("fp32 inputs: kernel_ms covers the bf16 hi/lo split and the contraction (3 bf16 "
                       "products per fp32 product); tflops counts 2 N V D, tensor_tflops the bf16 products")
    del t, H, W, y
    torch.cuda.empty_cache()
    return res, (Hn, Wn, yn)


def time_e2e(flce, fwd, H_h, W_h, y_h, w, dev, stream, args, world, mean_loss):
    """End to end: the forward with its inputs in pinned host memory, through
    flce_forward_host (bf16), and with the head resident on the device."""
    import torch
    N, V, D = w.N, w.V, w.D
    H, W = fwd.H, fwd.W
    host_ws = None
    if w.dtype == "bf16":
        host_ws = torch.empty(flce.host_workspace_size(N, V, D), dtype=torch.uint8, device=dev)
        copy_stream = torch.cuda.Stream(dev)
        res_h = {k: torch.empty(N, pin_memory=True) for k in ("loss", "lse", "target_logit")}
        res_h["mean"] = torch.empty((), pin_memory=True)
        mean_h = res_h["mean"]

        def e2e_step():
            flce.forward_host(H_h, W_h, y_h, device=dev, out=res_h, workspace=host_ws,
                              stream=stream, copy_stream=copy_stream)
        d2h = 3 * N * 4 + 4
    else:
        H_d2, W_d2, y_d2 = torch.empty_like(H), torch.empty_like(W), torch.empty_like(fwd.y)
        loss_h = torch.empty(N, pin_memory=True)
        mean_h = torch.empty((), pin_memory=True)
        out2 = {"loss": torch.empty(N, device=dev), "lse": torch.empty(N, device=dev),
                "target_logit": torch.empty(N, device=dev), "mean": torch.empty((), device=dev)}

        def e2e_step():
            H_d2.copy_(H_h, non_blocking=True)
            W_d2.copy_(W_h, non_blocking=True)
            y_d2.copy_(y_h, non_blocking=True)
            flce.forward(H_d2, W_d2, y_d2, out=out2, workspace=fwd.ws, stream=stream)
            loss_h.copy_(out2["loss"], non_blocking=True)
            mean_h.copy_(out2["mean"], non_blocking=True)
        d2h = N * 4 + 4

    def timed(fn, steps):
        import torch.distributed as dist
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
            stream.synchronize()
            if world > 1:
                dist.barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(steps):
                fn()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / steps

    Ke = max(3, min(args.steps, args.e2e_steps))
    e2e_ms = timed(e2e_step, Ke)
    if host_ws is not None and flce.check(host_ws, stream) != flce.OK:
        raise flce.FlceError(flce.check(host_ws, stream), "forward_host")
    assert abs(float(mean_h.item()) - mean_loss) <= 1e-5 * abs(mean_loss)
    h2d = H_h.numel() * H_h.element_size() + W_h.numel() * W_h.element_size() + y_h.numel() * 8

    # the head resident on the device (a parameter): H and y copied in and the
    # results out every step, around flce_forward
    H_r, y_r = torch.empty_like(H), torch.empty_like(fwd.y)
    res_r = {k: torch.empty(N, pin_memory=True) for k in ("loss", "lse", "target_logit")}
    res_r["mean"] = torch.empty((), pin_memory=True)
    out_r = {"loss": torch.empty(N, device=dev), "lse": torch.empty(N, device=dev),
             "target_logit": torch.empty(N, device=dev), "mean": torch.empty((), device=dev)}

    def resident_step():
        H_r.copy_(H_h, non_blocking=True)
        y_r.copy_(y_h, non_blocking=True)
        flce.forward(H_r, W, y_r, out=out_r, workspace=fwd.ws, stream=stream)
        for k in res_r:
            res_r[k].copy_(out_r[k], non_blocking=True)

    resident_ms = timed(resident_step, Ke)
    assert abs(float(res_r["mean"].item()) - mean_loss) <= 1e-6 * abs(mean_loss)
    e2e_ms, resident_ms = max_over_ranks([e2e_ms, resident_ms], world, device=dev)
    return {"e2e": {"value": weak_scaling_tokens_per_s(world, N, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms,
                    "steps": Ke,
                    "api": "flce_forward_host" if host_ws is not None else "torch copies + flce_forward"},
            "resident": {"value": weak_scaling_tokens_per_s(world, N, resident_ms), "unit": "tokens/s",
                         "h2d_bytes_per_step": int(H_h.numel() * H_h.element_size() + y_h.numel() * 8),
                         "d2h_bytes_per_step": int(3 * N * 4 + 4), "ms_per_step": resident_ms,
                         "what": "W resident on the device (a parameter); H and y copied in and the "
                                 "results out every step, around flce_forward"}}


def time_backward(flce, H, W, y, lse, N, V, D, dev, stream, args, peaks, world, gpu_index=0):
    """The backward (dH, dW of the mean loss) on the same inputs: per-step events over
    at least --backward-steps steps and about 1.5 s, with the SM clock sampled, so that
    its rate per MHz compares with the forward's sustained window."""
    import torch
    out = {"dH": torch.empty(N, D, device=dev), "dW": torch.empty(V, D, device=dev)}
    ws = torch.empty(flce.backward_workspace_size(N, V, D, H.dtype), dtype=torch.uint8, device=dev)

    def step():
        flce.backward(H, W, y, lse, None, 1.0 / N, out=out, workspace=ws, stream=stream)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(2):
            step()
        e0.record(stream)
        step()
        e1.record(stream)
    stream.synchronize()
    if flce.check(ws, stream) != flce.OK:
        raise flce.FlceError(flce.check(ws, stream), "backward")
    Kb = max(3, args.backward_steps, int(1500.0 / max(e0.elapsed_time(e1), 1e-3)))
    Kb = int(max_over_ranks([Kb], world, device=dev)[0])   # the same step count on every rank
    sampler = ClockSampler(gpu_index)
    sampler.start()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Kb)]
    t0 = time.time()
    with torch.cuda.stream(stream):
        for k in range(Kb):
            ev[k][0].record(stream)
            step()
            ev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    t1 = time.time()
    sampler.stop()
    per = [ev[k][0].elapsed_time(ev[k][1]) for k in range(Kb)]
    ms, ms_mean = max_over_ranks([median(per), float(np.mean(per))], world, device=dev)
    flops = 3 * 2 * N * V * D          # logits regenerated, dH, dW
    tflops = flops / (ms * 1e-3) / 1e12
    res = {"ms_per_step": ms, "ms_per_step_mean": ms_mean, "steps": Kb,
           "tokens_per_s": weak_scaling_tokens_per_s(world, N, ms),
           "flops_per_step": flops, "tflops": tflops, "frac_of_bf16_peak": tflops / peaks["bf16_tflops"],
           "frac_of_sustained_peak": tflops / peaks["bf16_tflops_sustained"],
           "workspace_bytes": int(ws.numel()),
           "what": "dH and dW of the mean loss from the forward's lse (3 contractions per step); "
                   "median of per-step events"}
    clocks = sampler.summary(t0, t1)
    if clocks:
        res["clocks"] = clocks
        res["tflops_per_mhz"] = tflops / clocks["sm_mhz"]
        res["frac_of_per_cycle_peak_at_median_clock"] = tflops / (
            B200_SMS * FLOP_PER_SM_CYCLE * clocks["sm_mhz"] * 1e6 / 1e12)
    return res


def time_quantized(flce, H, Wn, y, N, V, D, bits, gs, dev, stream, args, peaks, world):
    """The forward with the workload's W quantised to `bits`-bit codes in groups of `gs`
    (affine, MLX layout), on the same H and y, timed like the forward; and its dH."""
    import torch
    wq, sc, bi = synth.quantize_affine(synth.bf16_bits_to_f32(Wn), bits, gs)
    wqd = torch.from_numpy(wq.view(np.int32)).to(dev)
    scd = torch.from_numpy(sc).view(torch.bfloat16).to(dev)
    bid = torch.from_numpy(bi).view(torch.bfloat16).to(dev)
    ws = torch.empty(flce.quantized_workspace_size(N, V, D, bits, gs), dtype=torch.uint8, device=dev)
    out = {"loss": torch.empty(N, device=dev), "lse": torch.empty(N, device=dev),
           "target_logit": torch.empty(N, device=dev), "mean": torch.empty((), device=dev)}

    def timed(fn, steps, ws_check, what):
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
        stream.synchronize()
        if flce.check(ws_check, stream) != flce.OK:
            raise flce.FlceError(flce.check(ws_check, stream), what)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        with torch.cuda.stream(stream):
            for k in range(steps):
                ev[k][0].record(stream)
                fn()
                ev[k][1].record(stream)
        torch.cuda.synchronize(dev)
        return max_over_ranks([median([ev[k][0].elapsed_time(ev[k][1]) for k in range(steps)])],
                              world, device=dev)[0]

    Kq = max(3, args.steps // 2)
    ms = timed(lambda: flce.forward_quantized(H, wqd, scd, bid, y, bits, gs, out=out, workspace=ws,
                                              stream=stream), Kq, ws, "forward_quantized")
    flops = 2 * N * V * D
    Ds = (D + 63) // 64 * 64
    tensor_flops = 2 * N * V * 2 * Ds      # H hi^T + H lo^T
    head_bytes = wq.nbytes + sc.nbytes + bi.nbytes
    bws = torch.empty(flce.backward_quantized_workspace_size(N, V, D, bits, gs), dtype=torch.uint8,
                      device=dev)
    dH = torch.empty(N, D, device=dev)
    Kb = max(3, args.backward_steps)
    bms = timed(lambda: flce.backward_quantized(H, wqd, scd, bid, y, out["lse"], None, 1.0 / N, bits, gs,
                                                out=dH, workspace=bws, stream=stream),
                Kb, bws, "backward_quantized")
    bflops = 2 * N * V * 2 * Ds + 2 * 2 * N * V * D   # logits H hi^T + H lo^T, dZ W_hi + dZ W_lo
    return {"bits": bits, "group_size": gs, "ms_per_step": ms, "steps": Kq,
            "tokens_per_s": weak_scaling_tokens_per_s(world, N, ms),
            "tflops": flops / (ms * 1e-3) / 1e12,
            "tensor_tflops": tensor_flops / (ms * 1e-3) / 1e12,
            "tensor_frac_of_bf16_peak": tensor_flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "head_bytes": int(head_bytes), "bf16_head_bytes": int(2 * V * D),
            "workspace_bytes": int(ws.numel()), "mean_loss": float(out["mean"].item()),
            "backward_ms_per_step": bms, "backward_tensor_tflops": bflops / (bms * 1e-3) / 1e12,
            "backward_what": "dH only (the quantised head is frozen): regenerated logits, 2 GEMMs",
            "what": "forward with an affine group-quantised head: W expanded per 16384-row chunk "
                    "to bf16 hi/lo, 2 bf16 products per weight; medians of per-step events"}


def time_fp32(flce, w, rank, y, dev, stream, args, peaks, world):
    """The forward and the backward on the same workload drawn in fp32: the samples the
    bf16 inputs are rounded from, kept as they are.  Each call splits H and W into bf16
    hi/lo parts and runs three bf16 products per fp32 product."""
    import torch
    N, V, D = w.N, w.V, w.D
    Hn, Wn, _ = synth.generate(dataclasses.replace(w, dtype="fp32"), token_stream=rank)
    H = torch.from_numpy(Hn).to(dev)
    W = torch.from_numpy(Wn).to(dev)
    del Hn, Wn
    ws = torch.empty(flce.workspace_size(N, V, D, torch.float32), dtype=torch.uint8, device=dev)
    out = {"loss": torch.empty(N, device=dev), "lse": torch.empty(N, device=dev),
           "target_logit": torch.empty(N, device=dev), "mean": torch.empty((), device=dev)}

    def timed(fn, steps, what, ws_check):
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
        stream.synchronize()
        if flce.check(ws_check, stream) != flce.OK:
            raise flce.FlceError(flce.check(ws_check, stream), what)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        with torch.cuda.stream(stream):
            for k in range(steps):
                ev[k][0].record(stream)
                fn()
                ev[k][1].record(stream)
        torch.cuda.synchronize(dev)
        if flce.check(ws_check, stream) != flce.OK:
            raise flce.FlceError(flce.check(ws_check, stream), what)
        return max_over_ranks([median([ev[k][0].elapsed_time(ev[k][1]) for k in range(steps)])],
                              world, device=dev)[0]

    Kf = max(3, args.steps // 4)
    ms = timed(lambda: flce.forward(H, W, y, out=out, workspace=ws, stream=stream), Kf,
               "forward (fp32)", ws)
    Dp = (D + 63) // 64 * 64
    tensor_flops = 2 * N * V * 3 * Dp          # hi hi + hi lo + lo hi per K block
    res = {"ms_per_step": ms, "steps": Kf, "tokens_per_s": weak_scaling_tokens_per_s(world, N, ms),
           "tflops": 2 * N * V * D / (ms * 1e-3) / 1e12,
           "tensor_tflops": tensor_flops / (ms * 1e-3) / 1e12,
           "tensor_frac_of_bf16_peak": tensor_flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
           "workspace_bytes": int(ws.numel()), "mean_loss": float(out["mean"].item()),
           "what": "fp32 H and W (the workload's samples before bf16 rounding): each call splits "
                   "them into bf16 hi/lo and runs 3 bf16 products per fp32 product; tflops counts "
                   "2 N V D, tensor_tflops the bf16 products; medians of per-step events"}
    bws = torch.empty(flce.backward_workspace_size(N, V, D, torch.float32), dtype=torch.uint8,
                      device=dev)
    grads = {"dH": torch.empty(N, D, device=dev), "dW": torch.empty(V, D, device=dev)}
    Kb = max(3, args.backward_steps // 2)
    bms = timed(lambda: flce.backward(H, W, y, out["lse"], None, 1.0 / N, out=grads,
                                      workspace=bws, stream=stream), Kb, "backward (fp32)", bws)
    Db = (D + 7) // 8 * 8
    btensor = 2 * N * V * 3 * Db + 2 * 3 * 2 * N * V * D    # logits over 3 segments; 3 + 3 products
    res.update({"backward_ms_per_step": bms, "backward_steps": Kb,
                "backward_tflops": 3 * 2 * N * V * D / (bms * 1e-3) / 1e12,
                "backward_tensor_tflops": btensor / (bms * 1e-3) / 1e12,
                "backward_workspace_bytes": int(bws.numel())})
    del bws, grads, H, W, ws
    torch.cuda.empty_cache()
    return res


def torch_materialised(H, W, y, dev):
    """The materialising forward (cuBLAS logits + logsumexp) timed the same way, for context."""
    import torch
    try:
        def f():
            Z = torch.matmul(H, W.t())                     # (N, V) bf16 logits
            lse = torch.logsumexp(Z.float(), dim=1)
            return lse - Z.gather(1, y[:, None]).float().squeeze(1)
        for _ in range(2):
            f()
        torch.cuda.synchronize(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        base = torch.cuda.memory_allocated(dev)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(5):
            f()
        e.record()
        torch.cuda.synchronize(dev)
        return {"torch_materialised_ms": s.elapsed_time(e) / 5,
                "torch_materialised_extra_gib": (torch.cuda.max_memory_allocated(dev) - base) / 2 ** 30}
    except RuntimeError as ex:  # out of memory on very large shapes
        return {"torch_materialised_error": str(ex)[:200]}


# ----------------------------------------------------------------------------- vocabulary-parallel arm

def vocab_parallel_legs(flce, H, W_shard, y, v_offset: int, V_total: int, world: int, steps: int,
                        warmup: int, backward: bool = True, group=None):
    """The vocabulary-parallel forward (and backward) of one rank, stage by stage.

    Forward step: this rank's shard state (flce_partials_shard + flce_shard_state,
    its own contraction), one all-gather of the (N, 4) fp32 states (16 bytes per
    token per rank), and the merge (flce_merge_shards) into loss, lse and mean for
    the whole vocabulary.  Backward step: backward_vocab_parallel (this shard's
    dW rows and dH share, then one all-reduce of the N x D fp32 dH, overlapped with
    the last dW GEMMs on a side stream).  Times each stage with events on the
    current stream (host clock on CPU tensors) and returns per-rank medians.
    """
    import torch
    import torch.distributed as dist
    dev = H.device
    N, D = H.shape
    Vs = W_shard.shape[0]
    new_event = event_factory(dev)
    ws = torch.empty(flce.workspace_size(N, Vs, D, H.dtype), dtype=torch.uint8, device=dev) \
        if dev.type == "cuda" else None
    gather = {}

    def fwd_step(ev):
        ev[0].record()
        state = flce.shard_state(H, W_shard, y, v_offset, workspace=ws) if ws is not None \
            else flce.shard_state(H, W_shard, y, v_offset)
        ev[1].record()
        if world > 1:
            if "flat" not in gather:
                gather["flat"] = torch.empty(world * N, 4, dtype=state.dtype, device=dev)
            dist.all_gather_into_tensor(gather["flat"], state.contiguous(), group=group)
            gathered = gather["flat"].view(world, N, 4)
        else:
            gathered = state.unsqueeze(0)
        ev[2].record()
        res = flce.merge_shards(gathered.contiguous(), y, V_total)
        ev[3].record()
        return res

    for _ in range(max(1, warmup)):
        res = fwd_step([new_event() for _ in range(4)])
    sync(dev)
    if world > 1:
        dist.barrier(group=group)
    evs = [[new_event() for _ in range(4)] for _ in range(steps)]
    for k in range(steps):
        res = fwd_step(evs[k])
    sync(dev)
    part = lambda a, b: [e[a].elapsed_time(e[b]) for e in evs]  # noqa: E731
    fw = {"compute_ms": median(part(0, 1)), "exchange_ms": median(part(1, 2)),
          "merge_ms": median(part(2, 3)), "ms_per_step": median(part(0, 3)),
          "exchange_bytes_per_rank": 16 * N * (world - 1),
          "what": "this rank's shard state, all-gather of 16 B per token per rank, merge"}
    out = {"forward": fw, "loss": res[0], "lse": res[1], "mean": res[3]}
    if backward:
        lse = res[1]

        def bwd_step(ev):
            ev[0].record()
            r = flce.backward_vocab_parallel(H, W_shard, y, lse, v_offset, V_total, grad_scale=1.0 / N,
                                             group=group)
            ev[1].record()
            return r

        bwd_step([new_event(), new_event()])
        sync(dev)
        if world > 1:
            dist.barrier(group=group)
        bev = [[new_event(), new_event()] for _ in range(max(1, steps // 2))]
        for e in bev:
            grads = bwd_step(e)
        sync(dev)
        bw = {"ms_per_step": median([e[0].elapsed_time(e[1]) for e in bev]),
              "exchange_bytes_per_rank": 4 * N * D * 2 * (world - 1) // max(1, world),
              "what": "this shard's dW rows and dH share; one all-reduce of the N x D fp32 dH on a "
                      "side stream, overlapped with the last dW GEMMs"}
        # the all-reduce alone, the same size, for the exchange's own cost
        if world > 1:
            buf = torch.zeros(N, D, dtype=grads[0].dtype, device=dev)
            e0, e1 = new_event(), new_event()
            dist.all_reduce(buf, group=group)
            sync(dev)
            e0.record()
            dist.all_reduce(buf, group=group)
            e1.record()
            sync(dev)
            bw["exchange_alone_ms"] = e0.elapsed_time(e1)
        out["backward"] = bw
        out["dH"], out["dW_shard"] = grads
    return out


def run_vocab(args, w, rank, world, local_rank):
    """`--parallel vocab`: W's rows split over the ranks, the same tokens on every rank."""
    import torch
    import torch.distributed as dist

    import linear_cross_entropy_bf16_b200 as flce
    from linear_cross_entropy_bf16_b200 import build as lib_build

    if rank == 0:
        lib_build.build()
    if world > 1:
        dist.barrier()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    flce.load_library()
    peaks, peak_kind = measured_peaks()
    Hn, Wn, yn = synth.generate(w)
    a, b = vocab_shard_bounds(w.V, world, rank)
    (H_h, _, y_h), (H, W_shard, y) = to_device_tensors(Hn, Wn[a:b], yn, dev, pin=True)
    del Wn
    with torch.cuda.stream(torch.cuda.Stream(dev)):
        res = vocab_parallel_legs(flce, H, W_shard, y, a, w.V, world, args.steps, args.warmup,
                                  backward="backward" in args.legs)
    fw = res["forward"]
    vals = [fw["ms_per_step"], fw["compute_ms"], fw["exchange_ms"], fw["merge_ms"]]
    if "backward" in res:
        vals += [res["backward"]["ms_per_step"], res["backward"].get("exchange_alone_ms", 0.0)]
    vals = max_over_ranks(vals, world, device=dev)
    # end to end: H and y from pinned host memory every step, results back
    loss_h, mean_h = torch.empty(w.N, pin_memory=True), torch.empty((), pin_memory=True)
    H2, y2 = torch.empty_like(H), torch.empty_like(y)

    def e2e_step():
        H2.copy_(H_h, non_blocking=True)
        y2.copy_(y_h, non_blocking=True)
        r = vocab_parallel_legs(flce, H2, W_shard, y2, a, w.V, world, 1, 0, backward=False)
        loss_h.copy_(r["loss"], non_blocking=True)
        mean_h.copy_(r["mean"], non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks([(time.perf_counter() - t0) / 3 * 1e3], world, device=dev)[0]
    if rank != 0:
        return 0
    ms = vals[0]
    shard_flops = 2 * w.N * (b - a) * w.D
    line = {
        "metric": METRIC, "value": w.N / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": w.N / (ms * 1e-3) / PAGES_TOKENS_PER_S,
        "dtype": "bf16", "data": "synthetic (seeded numpy: H~N(0,1), W~N(0,1/D), targets per workload)",
        "config": workload_config(w, world, "vocab"),
        "roofline": {"bound": "tensor", "kernel": "flce_tc2_kernel (one shard)",
                     "achieved": shard_flops / (vals[1] * 1e-3) / 1e12, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": shard_flops / (vals[1] * 1e-3) / 1e12 / peaks["bf16_tflops"],
                     "peak_kind": f"{peak_kind} burst bf16", "traffic": None,
                     "kernel_ms": vals[1], "flops_per_launch": shard_flops},
        "vocab_parallel": {"forward": {**res["forward"], "ms_per_step": vals[0], "compute_ms": vals[1],
                                       "exchange_ms": vals[2], "merge_ms": vals[3]},
                           **({"backward": {**res["backward"], "ms_per_step": vals[4],
                                            "exchange_alone_ms": vals[5]}} if "backward" in res else {}),
                           "shard_rows_rank0": [a, b]},
        "e2e": {"value": w.N / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(H_h.numel() * 2 + y_h.numel() * 8),
                "d2h_bytes_per_step": int(w.N * 4 + 4), "ms_per_step": e2e_ms,
                "what": "W shards resident; H and y copied in and loss, mean out every step (host clock)"},
        "gpu_launches": 4 * args.steps,  # per step: header clear, contraction, shard state, merge
        "mean_loss": float(res["mean"].item()),
        "env": run_environment(dev),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=synth.HEADLINE, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--parallel", default="token", choices=["token", "vocab"],
                    help="token: each rank its own batch, W replicated (default); "
                         "vocab: W's rows split over the ranks, one all-gather per step")
    ap.add_argument("--legs", default=",".join(ALL_LEGS),
                    help=f"comma-separated subset of {','.join(ALL_LEGS)}, or 'none'")
    ap.add_argument("--sustain-seconds", type=float, default=3.0,
                    help="length of the sustained window the roofline's median kernel time comes from")
    ap.add_argument("--cpu-rows", type=int, default=256,
                    help="rows of each large workload the CPU oracle computes (all rows when N is smaller)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward-steps", type=int, default=10)
    ap.add_argument("--quantized", default="4,64", metavar="BITS,GROUP",
                    help="code width and group size of the quantised-head leg")
    ap.add_argument("--context", action="store_true", help="also time the materialising torch forward")
    ap.add_argument("--shape", default=None,
                    help="N,V,D: a custom shape with the chosen workload's distributions "
                         "(used for small profiling captures; not a reported workload)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    args.legs = [] if args.legs.strip() in ("", "none") else [s.strip() for s in args.legs.split(",")]
    unknown = set(args.legs) - set(ALL_LEGS)
    if unknown:
        ap.error(f"unknown legs: {sorted(unknown)}")
    w = synth.WORKLOADS[args.workload]
    if args.shape:
        n, v, d = (int(x) for x in args.shape.split(","))
        w = synth.Workload(f"custom_n{n}_v{v}_d{d}", n, v, d, w.dtype, w.targets, w.w_scale, w.seed)
        args.legs = [leg for leg in args.legs if leg != "workloads"]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        log(f"note: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE")

    if args.impl == "reference":
        return run_reference(args, w, rank, world)

    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.parallel == "vocab":
            return run_vocab(args, w, rank, world, local_rank)
        return run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
