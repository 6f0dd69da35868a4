#!/usr/bin/env python
"""Benchmark of the fused linear cross-entropy forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one full forward (contraction with online log-sum-exp, merge, mean)
over one batch of synthetic input already resident in HBM.  Rank 0 prints one
JSON line.  Under torchrun (N > 1) every rank runs its own batch of N tokens
against the same W (data-parallel, no collective on the data path; scaling is
weak) and the step time is the maximum over ranks.

Also measured: the contraction kernel's own duration (CUDA events around
flce_partials on the launching stream) for the roofline, an end-to-end leg
through the C ABI from pinned host buffers (flce_forward_host: H, y and W
copied in every step, W in chunks that overlap the contraction; results
copied back), SM clocks during the timed
region, and the CPU oracle on a bounded sample of the same workload.

Optional legs, each added to the same line as its own object: ``--backward``
(dH and dW), ``--quantized BITS,GROUP`` (a quantised head, with its dH when
``--backward`` is given too) and ``--fp32`` (the same workload's fp32 samples,
not rounded to bf16: forward, and backward with ``--backward``).

``--impl reference`` times the fp64 CPU oracle instead (the reference arm).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
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


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        # the raw samples go to FLCE_BENCH_CLOCKS_DIR when set (to keep them), else a temp file
        out_dir = os.environ.get("FLCE_BENCH_CLOCKS_DIR")
        self.path = os.path.join(out_dir, f"clocks_rank{gpu_index}.csv") if out_dir \
            else os.path.join(tempfile.gettempdir(), f"flce_clocks_{os.getpid()}_{gpu_index}.csv")
        self.gpu_index = gpu_index

    def start(self):
        if shutil.which("nvidia-smi") is None:
            return
        self.f = open(self.path, "w")
        self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                                      "--format=csv,noheader,nounits", "-lms", "100"],
                                     stdout=self.f, stderr=subprocess.DEVNULL)
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:9]))
            except ValueError:
                continue
        if not rows:
            return None
        sm = [r[0] for r in rows]
        loaded = [r for r in rows if r[2] > 300] or rows     # samples drawing real power
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3][1:]) if v.lower() == "active"})
        return {"sm_mhz": float(np.median([r[0] for r in loaded])), "sm_max_mhz": max(r[1] for r in rows),
                "sm_mhz_min": min(sm), "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(r[2] for r in rows), "reasons": reasons}


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


# ----------------------------------------------------------------------------- CPU oracle

def oracle_sample(H, W, y, seconds: float, seed: int, max_rows: int = 4096):
    """Time the oracle on growing batches of seeded rows until `seconds` have passed."""
    import oracle
    oracle.build()
    cores = oracle.max_threads()
    order = np.random.default_rng([seed, 99]).permutation(H.shape[0])
    done, t_total = 0, 0.0
    while t_total < seconds and done < min(max_rows, H.shape[0]):
        rows = order[done:done + cores]
        t0 = time.perf_counter()
        oracle.forward(H, W, y, rows=rows)
        t_total += time.perf_counter() - t0
        done += len(rows)
    return done, t_total, cores


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
        "scaling": "weak", "vs_baseline": value / PAGES_TOKENS_PER_S, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": w.name, "N": w.N, "V": w.V, "D": w.D, "input_dtype": w.dtype,
                   "targets": w.targets, "seed": w.seed, "global_batch": w.N, "parallelism": "none (host cores)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{per_step} seeded rows per step of the {w.name} workload "
                                   f"({rows} rows over {args.steps} steps); fp64, logits materialised per row"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm

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

    # inputs: W is the shared projection; each rank has its own tokens and targets
    t0 = time.perf_counter()
    Hn, Wn, yn = rank_inputs(w, rank)
    log(f"[rank {rank}] generated inputs in {time.perf_counter() - t0:.1f} s")

    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def host_tensor(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return t.view(torch.bfloat16) if a.dtype == np.uint16 else t

    H_h = host_tensor(Hn).pin_memory()
    W_h = host_tensor(Wn).pin_memory()
    y_h = torch.from_numpy(yn).pin_memory()
    H = H_h.to(dev)
    W = W_h.to(dev)
    y = y_h.to(dev)
    N, V, D = w.N, w.V, w.D
    ws = torch.empty(flce.workspace_size(N, V, D, tdt), dtype=torch.uint8, device=dev)
    loss = torch.empty(N, device=dev)
    lse = torch.empty(N, device=dev)
    tgt = torch.empty(N, device=dev)
    mean = torch.empty((), device=dev)
    out = {"loss": loss, "lse": lse, "target_logit": tgt, "mean": mean}
    stream = torch.cuda.Stream(dev)

    def step():
        flce.forward(H, W, y, out=out, workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
    stream.synchronize()
    st = flce.check(ws, stream)
    if st != flce.OK:
        raise flce.FlceError(st, "warm-up")

    # ---- timed region: K steps, per-kernel events on the launching stream
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    sampler = ClockSampler(local_rank)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for k in range(K):
            ev[k][0].record(stream)
            flce.partials(H, W, y, tgt, ws, stream=stream)
            ev[k][1].record(stream)
            flce.merge(y, V, loss, lse, tgt, mean, ws, stream=stream)
            ev[k][2].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = ev[0][0].elapsed_time(ev[K - 1][2])
    part_ms = [ev[k][0].elapsed_time(ev[k][1]) for k in range(K)]
    merge_ms = [ev[k][1].elapsed_time(ev[k][2]) for k in range(K)]
    st = flce.check(ws, stream)
    if st != flce.OK:
        raise flce.FlceError(st, "timed region")
    mean_loss = float(mean.item())

    # ---- end to end through the public API from pinned host memory:
    # flce_forward_host copies H and y, streams W in chunks (overlapping the
    # copies with the contraction) and copies the results back, every step
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
        H_d2 = torch.empty_like(H)
        W_d2 = torch.empty_like(W)
        y_d2 = torch.empty_like(y)
        loss_h = torch.empty(N, pin_memory=True)
        mean_h = torch.empty((), pin_memory=True)
        out2 = {"loss": torch.empty(N, device=dev), "lse": torch.empty(N, device=dev),
                "target_logit": torch.empty(N, device=dev), "mean": torch.empty((), device=dev)}

        def e2e_step():
            H_d2.copy_(H_h, non_blocking=True)
            W_d2.copy_(W_h, non_blocking=True)
            y_d2.copy_(y_h, non_blocking=True)
            flce.forward(H_d2, W_d2, y_d2, out=out2, workspace=ws, stream=stream)
            loss_h.copy_(out2["loss"], non_blocking=True)
            mean_h.copy_(out2["mean"], non_blocking=True)
        d2h = N * 4 + 4

    Ke = max(3, min(K, args.e2e_steps))
    with torch.cuda.stream(stream):
        for _ in range(3):
            e2e_step()
        stream.synchronize()
        if host_ws is not None and flce.check(host_ws, stream) != flce.OK:
            raise flce.FlceError(flce.check(host_ws, stream), "forward_host")
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(Ke):
            e2e_step()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / Ke
    assert abs(float(mean_h.item()) - mean_loss) <= 1e-5 * abs(mean_loss)
    h2d = H_h.numel() * H_h.element_size() + W_h.numel() * W_h.element_size() + y_h.numel() * 8

    # ---- the same with the head resident on the device (a training or
    # inference step, where W is a parameter): H and y copied in from pinned
    # host memory, the results copied out, every step
    H_r = torch.empty_like(H)
    y_r = torch.empty_like(y)
    res_r = {k: torch.empty(N, pin_memory=True) for k in ("loss", "lse", "target_logit")}
    res_r["mean"] = torch.empty((), pin_memory=True)
    out_r = {"loss": torch.empty(N, device=dev), "lse": torch.empty(N, device=dev),
             "target_logit": torch.empty(N, device=dev), "mean": torch.empty((), device=dev)}

    def resident_step():
        H_r.copy_(H_h, non_blocking=True)
        y_r.copy_(y_h, non_blocking=True)
        flce.forward(H_r, W, y_r, out=out_r, workspace=ws, stream=stream)
        for k in res_r:
            res_r[k].copy_(out_r[k], non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(3):
            resident_step()
        stream.synchronize()
        if world > 1:
            dist.barrier()
        e0.record(stream)
        for _ in range(Ke):
            resident_step()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    resident_ms = e0.elapsed_time(e1) / Ke
    assert abs(float(res_r["mean"].item()) - mean_loss) <= 1e-6 * abs(mean_loss)

    # ---- max over ranks
    resident_ms = max_over_ranks([resident_ms], world, device=dev)[0]
    total_ms, part_avg_ms, e2e_ms = max_over_ranks([total_ms, float(np.mean(part_ms)), e2e_ms],
                                                   world, device=dev)

    # the optional legs take their own max over ranks: every rank runs them
    peaks, peak_kind = measured_peaks()
    extra = {}
    if args.backward and w.dtype == "bf16":
        extra["backward"] = time_backward(flce, H, W, y, lse, N, V, D, tdt, dev, stream, args,
                                          peaks["bf16_tflops"], world)
    if args.quantized and w.dtype == "bf16":
        bits, gs = (int(v) for v in args.quantized.split(","))
        extra["quantized"] = time_quantized(flce, H, Wn, y, N, V, D, bits, gs, dev, stream, args,
                                            peaks["bf16_tflops"], world)
    if args.fp32 and w.dtype == "bf16":
        extra["fp32"] = time_fp32(flce, w, rank, y, dev, stream, args, peaks["bf16_tflops"], world)

    if rank != 0:
        return 0

    ms_step = total_ms / K
    tokens_per_s = weak_scaling_tokens_per_s(world, N, ms_step)
    flops = w.flops
    achieved = flops / (part_avg_ms * 1e-3) / 1e12
    p = flce.plan(N, V, D, tdt)
    # fp32 inputs run on the same kernels after the bf16 hi/lo split (three
    # bf16 products per fp32 product); `achieved` still counts 2 N V D.
    kernel = "flce_tc2_kernel" if p["ctas_per_unit"] == 2 else "flce_tc_kernel"
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
        "config": {"workload": w.name, "N": N, "V": V, "D": D, "input_dtype": w.dtype,
                   "targets": w.targets, "seed": w.seed, "global_batch": world * N,
                   "parallelism": f"dp{world}" if world > 1 else "single GPU",
                   "l2": f"inputs larger than L2 (W is {Wn.nbytes / 1e9:.2f} GB), no flush",
                   "tflops_per_gpu": flops / (ms_step / 1e3) / 1e12,
                   "frac_of_bf16_peak_per_gpu": flops / (ms_step / 1e3) / 1e12 / peaks["bf16_tflops"],
                   "mean_loss": mean_loss},
        "roofline": {"bound": "tensor", "kernel": kernel,
                     "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"],
                     "peak_kind": f"{peak_kind} burst bf16 (MEASURED_PEAKS.json bf16_tflops)",
                     "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                     "kernel_ms": part_avg_ms, "merge_ms": float(np.mean(merge_ms)),
                     "flops_per_launch": flops,
                     "traffic": profiled_traffic(w.name, kernel)},
        "e2e": {"value": weak_scaling_tokens_per_s(world, N, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms,
                "api": "flce_forward_host" if host_ws is not None else "torch copies + flce_forward"},
        "e2e_resident_head": {"value": weak_scaling_tokens_per_s(world, N, resident_ms), "unit": "tokens/s",
                              "h2d_bytes_per_step": int(H_h.numel() * H_h.element_size() + y_h.numel() * 8),
                              "d2h_bytes_per_step": int(3 * N * 4 + 4), "ms_per_step": resident_ms,
                              "what": "W resident on the device (a parameter); H and y copied in and the "
                                      "results out every step, around flce_forward"},
        "gpu_launches": 2 * K,
        "kernel_ms_stats": {"median": float(np.median(part_ms)), "min": float(np.min(part_ms)),
                            "max": float(np.max(part_ms))},
        "env": run_environment(dev),
        "clocks": clocks,
    }
    line.update(extra)
    if world == 1 and not args.no_cpu_baseline:
        rows, secs, cores = oracle_sample(Hn, Wn, yn, args.cpu_seconds, w.seed)
        line["cpu_baseline"] = {"value": rows / secs, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": f"{rows} seeded rows of {w.name} (full V and D per row), {secs:.1f} s"}
    if world == 1 and args.context:
        line["context"] = torch_materialised(H, W, y, dev)
    print(json.dumps(line), flush=True)
    return 0


def time_backward(flce, H, W, y, lse, N, V, D, tdt, dev, stream, args, peak, world):
    """The backward (dH, dW of the mean loss) on the same inputs, timed like the forward."""
    import torch
    out = {"dH": torch.empty(N, D, device=dev), "dW": torch.empty(V, D, device=dev)}
    ws = torch.empty(flce.backward_workspace_size(N, V, D, tdt), dtype=torch.uint8, device=dev)

    def step():
        flce.backward(H, W, y, lse, None, 1.0 / N, out=out, workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(3):
            step()
    stream.synchronize()
    if flce.check(ws, stream) != flce.OK:
        raise flce.FlceError(flce.check(ws, stream), "backward")
    Kb = max(3, args.backward_steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(Kb):
            step()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks([e0.elapsed_time(e1) / Kb], world, device=dev)[0]
    flops = 3 * 2 * N * V * D          # logits regenerated, dH, dW
    tflops = flops / (ms * 1e-3) / 1e12
    return {"ms_per_step": ms, "steps": Kb, "tokens_per_s": weak_scaling_tokens_per_s(world, N, ms),
            "flops_per_step": flops, "tflops": tflops, "frac_of_bf16_peak": tflops / peak,
            "workspace_bytes": int(ws.numel()),
            "what": "dH and dW of the mean loss from the forward's lse (3 contractions per step)"}


def time_quantized(flce, H, Wn, y, N, V, D, bits, gs, dev, stream, args, peak, world):
    """The forward with the workload's W quantised to `bits`-bit codes in groups of `gs`
    (affine, MLX layout), on the same H and y, timed like the forward."""
    import torch
    wq, sc, bi = synth.quantize_affine(synth.bf16_bits_to_f32(Wn), bits, gs)
    wqd = torch.from_numpy(wq.view(np.int32)).to(dev)
    scd = torch.from_numpy(sc).view(torch.bfloat16).to(dev)
    bid = torch.from_numpy(bi).view(torch.bfloat16).to(dev)
    ws = torch.empty(flce.quantized_workspace_size(N, V, D, bits, gs), dtype=torch.uint8, device=dev)
    out = {"loss": torch.empty(N, device=dev), "lse": torch.empty(N, device=dev),
           "target_logit": torch.empty(N, device=dev), "mean": torch.empty((), device=dev)}

    def step():
        flce.forward_quantized(H, wqd, scd, bid, y, bits, gs, out=out, workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
    stream.synchronize()
    if flce.check(ws, stream) != flce.OK:
        raise flce.FlceError(flce.check(ws, stream), "forward_quantized")
    Kq = max(3, args.steps // 2)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(Kq):
            step()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks([e0.elapsed_time(e1) / Kq], world, device=dev)[0]
    flops = 2 * N * V * D
    Ds = (D + 63) // 64 * 64
    tensor_flops = 2 * N * V * 2 * Ds      # H hi^T + H lo^T
    head_bytes = wq.nbytes + sc.nbytes + bi.nbytes
    extra = {}
    if args.backward:
        # dH of the mean loss for the frozen quantised head
        bws = torch.empty(flce.backward_quantized_workspace_size(N, V, D, bits, gs),
                          dtype=torch.uint8, device=dev)
        dH = torch.empty(N, D, device=dev)

        def bstep():
            flce.backward_quantized(H, wqd, scd, bid, y, out["lse"], None, 1.0 / N, bits, gs,
                                    out=dH, workspace=bws, stream=stream)
        with torch.cuda.stream(stream):
            for _ in range(3):
                bstep()
        stream.synchronize()
        if flce.check(bws, stream) != flce.OK:
            raise flce.FlceError(flce.check(bws, stream), "backward_quantized")
        Kb = max(3, args.backward_steps)
        e0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(Kb):
                bstep()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        bms = max_over_ranks([e0.elapsed_time(e1) / Kb], world, device=dev)[0]
        bflops = 2 * N * V * 2 * Ds + 2 * 2 * N * V * D   # logits H hi^T + H lo^T, dZ W_hi + dZ W_lo
        extra = {"backward_ms_per_step": bms, "backward_tensor_tflops": bflops / (bms * 1e-3) / 1e12,
                 "backward_what": "dH only (the quantised head is frozen): regenerated logits, 2 GEMMs"}
    return {**extra, "bits": bits, "group_size": gs, "ms_per_step": ms, "steps": Kq,
            "tokens_per_s": weak_scaling_tokens_per_s(world, N, ms),
            "tflops": flops / (ms * 1e-3) / 1e12,
            "tensor_tflops": tensor_flops / (ms * 1e-3) / 1e12,
            "tensor_frac_of_bf16_peak": tensor_flops / (ms * 1e-3) / 1e12 / peak,
            "head_bytes": int(head_bytes), "bf16_head_bytes": int(2 * V * D),
            "workspace_bytes": int(ws.numel()), "mean_loss": float(out["mean"].item()),
            "what": "forward with an affine group-quantised head: W expanded per 16384-row chunk "
                    "to bf16 hi/lo, 2 bf16 products per weight"}


def time_fp32(flce, w, rank, y, dev, stream, args, peak, world):
    """The forward (and with --backward the backward) on the same workload drawn in fp32:
    the samples the bf16 inputs are rounded from, kept as they are.  Each call splits H
    and W into bf16 hi/lo parts and runs three bf16 products per fp32 product."""
    import dataclasses

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
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(steps):
                fn()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        if flce.check(ws_check, stream) != flce.OK:
            raise flce.FlceError(flce.check(ws_check, stream), what)
        return max_over_ranks([e0.elapsed_time(e1) / steps], world, device=dev)[0]

    Kf = max(3, args.steps // 5)
    ms = timed(lambda: flce.forward(H, W, y, out=out, workspace=ws, stream=stream), Kf,
               "forward (fp32)", ws)
    Dp = (D + 63) // 64 * 64
    tensor_flops = 2 * N * V * 3 * Dp          # hi hi + hi lo + lo hi per K block
    res = {"ms_per_step": ms, "steps": Kf, "tokens_per_s": weak_scaling_tokens_per_s(world, N, ms),
           "tflops": 2 * N * V * D / (ms * 1e-3) / 1e12,
           "tensor_tflops": tensor_flops / (ms * 1e-3) / 1e12,
           "tensor_frac_of_bf16_peak": tensor_flops / (ms * 1e-3) / 1e12 / peak,
           "workspace_bytes": int(ws.numel()), "mean_loss": float(out["mean"].item()),
           "what": "fp32 H and W (the workload's samples before bf16 rounding): each call splits "
                   "them into bf16 hi/lo and runs 3 bf16 products per fp32 product; tflops counts "
                   "2 N V D, tensor_tflops the bf16 products"}
    if args.backward:
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
        del bws, grads
    del H, W, ws
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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=synth.HEADLINE, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="also time the backward (dH, dW) and add a 'backward' object to the line")
    ap.add_argument("--backward-steps", type=int, default=10)
    ap.add_argument("--quantized", default=None, metavar="BITS,GROUP",
                    help="also time the forward with W quantised (e.g. 4,64) and add a 'quantized' object")
    ap.add_argument("--context", action="store_true", help="also time the materialising torch forward")
    ap.add_argument("--fp32", action="store_true",
                    help="also time the forward (and with --backward the backward) on the workload's "
                         "fp32 samples and add an 'fp32' object")
    ap.add_argument("--shape", default=None,
                    help="N,V,D: a custom shape with the chosen workload's distributions "
                         "(used for small profiling captures; not a reported workload)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = synth.WORKLOADS[args.workload]
    if args.shape:
        n, v, d = (int(x) for x in args.shape.split(","))
        w = synth.Workload(f"custom_n{n}_v{v}_d{d}", n, v, d, w.dtype, w.targets, w.w_scale, w.seed)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        log(f"note: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE")

    if args.impl == "reference":
        return run_reference(args, w, rank, world)

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
