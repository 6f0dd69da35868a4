"""A seeded sweep of random problem shapes through the forward entry points,
every row against the oracle.  The shapes (ragged N, V and D, bf16 and fp32,
int32 and int64 targets, strided rows, quantised heads) are drawn once from a
fixed seed, so the sweep is the same on every run."""
import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_bf16_b200 import synth
from tests.flce_testing import compare, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_cross_entropy_bf16_b200 import build
    build.build()
    oracle.build()


def draw_cases(n=24, seed=2026, budget=4e9):
    rng = np.random.default_rng(seed)
    cases = []
    while len(cases) < n:
        dtype = "fp32" if rng.random() < 0.35 else "bf16"
        N = int(rng.choice([1, 2, 127, 128, 129, 255, 256, 257, 300, 511, 700, 1000]))
        V = int(np.exp(rng.uniform(0.0, np.log(40000.0))))          # log-uniform in [1, 40000]
        D = int(rng.integers(1, 97)) * 8 if dtype == "bf16" else int(rng.integers(1, 300))
        if N * V * D > budget:
            continue
        pad = int(rng.integers(0, 3)) * 8        # row padding: strided H and W when > 0
        y32 = bool(rng.random() < 0.5)
        cases.append((dtype, N, V, D, pad, y32))
    return cases


@pytest.mark.parametrize("dtype,N,V,D,pad,y32", draw_cases())
def test_random_shapes_every_row(dtype, N, V, D, pad, y32):
    import linear_cross_entropy_bf16_b200 as flce
    H, W, y = synth.random_inputs(N, V, D + pad, seed=N * 31 + V + D, dtype=dtype)
    Hd, Wd, yd = to_device(H, W, y)
    if y32:
        yd = yd.to(torch.int32)
    Hs, Ws = Hd[:, pad:], Wd[:, :D]
    loss, lse, tgt, mean = flce.forward_strided(Hs, Ws, yd, check=True)
    Hc, Wc = np.ascontiguousarray(H[:, pad:]), np.ascontiguousarray(W[:, :D])
    ref = oracle.forward(Hc, Wc, y)
    gpu = {"loss": loss.cpu().double().numpy(), "lse": lse.cpu().double().numpy(),
           "target": tgt.cpu().double().numpy(), "mean": float(mean.item())}
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))


def draw_quantized(n=6, seed=2027):
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < n:
        bits = int(rng.choice([2, 4, 8]))
        G = int(rng.choice([32, 64, 128]))
        D = G * int(rng.integers(1, 5))
        N = int(rng.choice([1, 100, 129, 300]))
        V = int(rng.integers(1, 40001))
        if N * V * D <= 1.5e9:
            out.append((N, V, D, bits, G))
    return out


@pytest.mark.parametrize("N,V,D,bits,G", draw_quantized())
def test_random_quantised_heads_every_row(N, V, D, bits, G):
    import linear_cross_entropy_bf16_b200 as flce
    H, Wf, y = synth.random_inputs(N, V, D, seed=N + V + D + bits, dtype="fp32")
    H = synth.round_to_bf16_bits(H)
    wq, sc, bi = synth.quantize_affine(Wf, bits, G)
    dev = torch.device("cuda:0")
    args = (torch.from_numpy(H).view(torch.bfloat16).to(dev), torch.from_numpy(wq.view(np.int32)).to(dev),
            torch.from_numpy(sc).view(torch.bfloat16).to(dev), torch.from_numpy(bi).view(torch.bfloat16).to(dev),
            torch.from_numpy(y).to(dev))
    loss, lse, tgt, mean = flce.forward_quantized(*args, bits, G, check=True)
    ref = oracle.forward_quantized(H, wq, sc, bi, y, bits, G)
    gpu = {"loss": loss.cpu().double().numpy(), "lse": lse.cpu().double().numpy(),
           "target": tgt.cpu().double().numpy(), "mean": float(mean.item())}
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))


def draw_backward(n=10, seed=2028, budget=1.2e9):
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < n:
        dtype = "fp32" if rng.random() < 0.4 else "bf16"
        N = int(rng.choice([1, 7, 128, 129, 256, 300, 513]))
        V = int(np.exp(rng.uniform(0.0, np.log(40000.0))))
        D = int(rng.integers(1, 49)) * 8 if dtype == "bf16" else int(rng.integers(1, 200))
        if N * V * D <= budget:
            out.append((dtype, N, V, D))
    return out


@pytest.mark.parametrize("dtype,N,V,D", draw_backward())
def test_random_shapes_backward_every_element(dtype, N, V, D):
    """dH and dW of sum_i g_i loss_i on every element, within 2^-8 of the oracle's
    magnitude bound (the bf16 rounding of dZ; fp32 inputs do far better)."""
    import linear_cross_entropy_bf16_b200 as flce
    H, W, y = synth.random_inputs(N, V, D, seed=3 * N + V + D, dtype=dtype)
    Hd, Wd, yd = to_device(H, W, y)
    _, lse, _, _ = flce.forward(Hd, Wd, yd, check=True)
    g = np.random.default_rng(N + V).uniform(-1, 1, N)
    gd = torch.from_numpy(g.astype(np.float32)).cuda()
    dH, dW = flce.backward(Hd, Wd, yd, lse, gd, 1.0, check=True)
    ref = oracle.backward(H, W, y, g.astype(np.float32).astype(np.float64), bounds=True)
    for got, r, b in ((dH, ref["dH"], ref["bH"]), (dW, ref["dW"], ref["bW"])):
        err = np.abs(got.cpu().double().numpy() - r)
        assert np.all(err <= 2.0 ** -8 * b + 1e-7), float((err - 2.0 ** -8 * b).max())
