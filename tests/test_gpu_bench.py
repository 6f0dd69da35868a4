"""The benchmark's JSON line on a GPU: one short run of `bench.py` (the N=1024,
V=32000, D=1024 workload, no optional legs) must print one line with every key
the run's consumers read, consistent with itself, and the reference arm must
print the same workload keys."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args):
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def test_bench_line_has_the_contract_keys():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    args = ["--workload", "n1024_v32000_d1024", "--legs", "none", "--steps", "4", "--warmup", "3",
            "--sustain-seconds", "0.5", "--e2e-steps", "3"]
    d = run_bench(*args)
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches",
              "clocks", "cpu_baseline", "sustained"):
        assert k in d, k
    assert d["steps"] == 4 and d["warmup"] == 3 and d["n_gpus"] == 1 and d["gpu_launches"] == 8
    assert d["value"] == pytest.approx(1024 / (d["ms_per_step"] * 1e-3), rel=1e-9)
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] > 0
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], rel=1e-9)
    assert r["achieved"] == pytest.approx(2 * 1024 * 32000 * 1024 / (r["kernel_ms"] * 1e-3) / 1e12,
                                          rel=1e-9)
    assert 0.05 < r["frac"] < 1.5            # a kernel that did the work, not a no-op
    e = d["e2e"]
    assert e["h2d_bytes_per_step"] >= 1024 * 1024 * 2 + 32000 * 1024 * 2 and e["d2h_bytes_per_step"] > 0
    assert e["value"] < d["value"]          # host copies inside the timed region
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["rows"] == 1024
    assert d["config"]["workload"] == "n1024_v32000_d1024" and "flushed" in d["config"]["l2"]
    ref = run_bench(*args[:2], "--impl", "reference", "--steps", "2", "--warmup", "3")
    assert ref["impl"] == "reference" and ref["config"] == d["config"]


def test_bench_vocab_parallel_mode_on_one_gpu():
    """`--parallel vocab` with one rank: the whole vocabulary is its shard, the
    exchange is empty, and the line reports each stage of the forward and the
    backward."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    d = run_bench("--workload", "n1024_v32000_d1024", "--parallel", "vocab", "--steps", "4", "--warmup", "3")
    assert d["scaling"] == "strong" and d["n_gpus"] == 1
    vp = d["vocab_parallel"]
    f = vp["forward"]
    assert f["compute_ms"] > 0 and f["merge_ms"] > 0 and f["exchange_bytes_per_rank"] == 0
    assert f["ms_per_step"] >= f["compute_ms"]
    assert vp["backward"]["ms_per_step"] > 0
    assert d["value"] == pytest.approx(1024 / (d["ms_per_step"] * 1e-3), rel=1e-9)
    assert 8.0 < d["mean_loss"] < 14.0     # about ln 32000 = 10.4 for logits of unit variance
