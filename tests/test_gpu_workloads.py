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

SAMPLE_ROWS = int(os.environ.get("FLCE_ORACLE_ROWS", "256"))


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


# ----------------------------------------------------------------------------- backward

def _backward(name, N=None, V=None, D=None):
    """dH and dW of the mean loss (device tensors), after checking bitwise repeatability."""
    import linear_cross_entropy_bf16_b200 as flce
    H, W, y = synth.generate(name, N=N, V=V, D=D)
    Hd, Wd, yd = to_device(H, W, y)
    _, lse, _, _ = flce.forward(Hd, Wd, yd, check=True)
    n = H.shape[0]
    dH, dW = flce.backward(Hd, Wd, yd, lse, None, 1.0 / n, check=True)
    again = flce.backward(Hd, Wd, yd, lse, None, 1.0 / n)
    assert torch.equal(dH, again[0]) and torch.equal(dW, again[1])
    return H, W, y, dH, dW


def _within(got, ref, bound):
    err = np.abs(got - ref)
    assert np.all(err <= 2.0 ** -8 * bound + 1e-7), float((err - 2.0 ** -8 * bound).max())


def test_backward_workload_n1024_every_element():
    """The N=1024, V=32000, D=1024 workload: every element of dH and dW (mean loss)."""
    H, W, y, dH, dW = _backward("n1024_v32000_d1024")
    g = np.float64(np.float32(1.0 / H.shape[0]))
    ref = oracle.backward(H, W, y, g, bounds=True)
    _within(dH.cpu().double().numpy(), ref["dH"], ref["bH"])
    _within(dW.cpu().double().numpy(), ref["dW"], ref["bW"])


def _dw_fixture(name, H, W, y):
    """The oracle's sampled dW rows for workload `name` (tests/golden/make_dw_rows.py),
    after checking that they were computed from these very inputs."""
    import hashlib
    path = os.path.join(os.path.dirname(__file__), "golden", f"dw_rows_{name}.npz")
    f = np.load(path)
    h = hashlib.sha256()
    for a in (H, W, y):
        h.update(np.ascontiguousarray(a).tobytes())
    assert str(f["input_sha256"]) == h.hexdigest(), "inputs differ from those the fixture was made from"
    return f


@pytest.mark.parametrize("name", [synth.HEADLINE, "n4096_v128256_d4096_zipf"])
def test_backward_full_size_dW_rows_every_element(name):
    """At full size the backward runs in several 32768-row vocabulary chunks; the
    sampled dW rows (chunk edges, the first and last rows, targets, seeded rows) are
    compared element by element with the oracle's (every token's lse recomputed in
    fp64), within the derived bound 2^-8 sum_i |dZ_ij| |H_ik|."""
    H, W, y, dH, dW = _backward(name)
    f = _dw_fixture(name, H, W, y)
    assert float(f["g"]) == float(np.float32(1.0 / H.shape[0]))
    rows = torch.from_numpy(f["vocab_rows"]).cuda()
    got = dW[rows].cpu().double().numpy()
    ref, bound = f["dW"].astype(np.float64), f["bW"].astype(np.float64)
    # dW entries here are ~1e-7 (g = 1/N), so no absolute slack: the bound alone
    err = np.abs(got - ref)
    assert np.all(err <= 2.0 ** -8 * bound + 1e-15), float((err / np.maximum(bound, 1e-300)).max())
    # and the comparison is not vacuous: the bound is small against the values
    assert np.median(2.0 ** -8 * bound / np.maximum(np.abs(ref), 1e-300)) < 1.0
    # the rows straddle the chunk edges of the backward
    edges = {int(r) % 32768 for r in f["vocab_rows"]}
    assert 0 in edges and 32767 in edges


def test_backward_headline_sampled_rows_and_properties():
    """The page's shape: sampled dH rows against the oracle; dW by its exact zero-sum."""
    H, W, y, dH, dW = _backward(synth.HEADLINE)
    w = synth.WORKLOADS[synth.HEADLINE]
    assert bool(torch.isfinite(dH).all()) and bool(torch.isfinite(dW).all())
    rows = synth.sample_rows(w.N, 16, w.seed)
    ref = oracle.grad_hidden_rows(H, W, y, np.float64(np.float32(1.0 / w.N)), rows)
    _within(dH[torch.from_numpy(rows).cuda()].cpu().double().numpy(), ref["dH"], ref["bH"])
    # sum_j dL/dZ_ij = 0 exactly, so the vocabulary rows of dW sum to zero up to the
    # bf16 rounding of dZ (relative 2^-9 per term); reduced on the device in fp64
    colsum = dW.double().sum(dim=0).abs().max().item()
    scale = dW.double().abs().sum(dim=0).max().item()
    assert colsum <= 2.0 ** -8 * scale
