"""The five measured workloads at full size, in the launch configuration the
benchmark times (one flce_forward call through the C ABI).

Small workloads are compared with the oracle on every row.  For the three
large ones the oracle computes a seeded sample of rows (always including the
first and last token), and properties that hold at any size are checked on
every row: finite values, loss >= 0, lse >= target logit, loss = lse - target
logit, the mean equal to the average of the per-token losses, and bitwise
determinism of a second call.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_bf16_b200 import synth
from tests.flce_testing import check_properties, compare, run, to_device

pytestmark = pytest.mark.gpu

SAMPLE_ROWS = int(os.environ.get("FLCE_ORACLE_ROWS", "128"))


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_cross_entropy_bf16_b200 import build
    build.build()
    oracle.build()


@pytest.mark.parametrize("name", ["tiny_n256_v2048_d256_fp32", "n1024_v32000_d1024"])
def test_small_workload_every_row(name):
    H, W, y = synth.generate(name)
    gpu = run(H, W, y)
    ref = oracle.forward(H, W, y)
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))
    check_properties(gpu, W.shape[0])


@pytest.mark.parametrize("name", ["n4096_v128256_d4096_zipf", "n8192_v151936_d4096",
                                  "stress_n16384_v262144_d2048"])
def test_large_workload_sampled_rows(name):
    import linear_cross_entropy_bf16_b200 as flce
    w = synth.WORKLOADS[name]
    H, W, y = synth.generate(name)
    Hd, Wd, yd = to_device(H, W, y)
    loss, lse, tgt, mean = flce.forward(Hd, Wd, yd, check=True)
    again = flce.forward(Hd, Wd, yd, check=True)
    for a, b in zip((loss, lse, tgt, mean), again):
        assert torch.equal(a, b)
    gpu = {"loss": loss.cpu().double().numpy(), "lse": lse.cpu().double().numpy(),
           "target": tgt.cpu().double().numpy(), "mean": float(mean.item())}
    check_properties(gpu, w.V)
    rows = synth.sample_rows(w.N, SAMPLE_ROWS, w.seed)
    ref = oracle.forward(H, W, y, rows=rows)
    compare(gpu, ref, rows=rows)
