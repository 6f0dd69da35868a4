"""GPU parity of the backward (dH, dW) against the fp64 oracle, through the C ABI.

Tolerance, derived from the arithmetic: dZ is rounded to bf16 (relative
error <= 2^-9) before the two contractions, which accumulate in fp32 over at
most K = 32768 (chunk) or N terms (error <= K 2^-24 <= 2^-9 of the magnitude), so
each entry satisfies |d dH_ik| <= 2^-8 sum_j |dZ_ij||W_jk| (the oracle's bH)
and |d dW_jk| <= 2^-8 sum_i |dZ_ij||H_ik| (bW) for the shapes below, plus a
tiny absolute floor for entries whose magnitude is zero.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_bf16_b200 import synth
from tests.flce_testing import to_device

pytestmark = pytest.mark.gpu
REL = 2.0 ** -8
FLOOR = 1e-7


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_cross_entropy_bf16_b200 import build
    build.build()
    oracle.build()


def run_backward(H, W, y, g=None, scale=1.0):
    import linear_cross_entropy_bf16_b200 as flce
    Hd, Wd, yd = to_device(H, W, y)
    _, lse, _, _ = flce.forward(Hd, Wd, yd, check=True)
    gd = torch.from_numpy(np.asarray(g, dtype=np.float32)).cuda() if g is not None else None
    dH, dW = flce.backward(Hd, Wd, yd, lse, gd, scale, check=True)
    torch.cuda.synchronize()
    return dH.cpu().double().numpy(), dW.cpu().double().numpy()


def compare(got, ref, bound, name):
    err = np.abs(got - ref)
    lim = REL * bound + FLOOR
    worst = np.unravel_index(np.argmax(err - lim), err.shape)
    assert np.all(np.isfinite(got)), name
    assert np.all(err <= lim), (f"{name}: |diff| {err[worst]:.3e} > {lim[worst]:.3e} at {worst} "
                                f"(gpu {got[worst]!r}, oracle {ref[worst]!r})")
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert rel < 3e-3, f"{name}: relative Frobenius error {rel:.2e}"
    return rel


SHAPES = [(1, 1, 8), (7, 3, 16), (130, 300, 64), (256, 1000, 128), (300, 2047, 72), (513, 777, 136),
          (64, 20000, 64), (1000, 600, 264)]


@pytest.mark.parametrize("N,V,D", SHAPES)
def test_backward_every_element(N, V, D):
    H, W, y = synth.random_inputs(N, V, D, seed=N + 3 * V + 7 * D)
    g = np.random.default_rng(N).uniform(-1, 1, N)
    dH, dW = run_backward(H, W, y, g)
    gf = g.astype(np.float32).astype(np.float64)       # the GPU receives fp32 g
    ref = oracle.backward(H, W, y, gf, bounds=True)
    compare(dH, ref["dH"], ref["bH"], "dH")
    compare(dW, ref["dW"], ref["bW"], "dW")


def test_backward_mean_loss_scale_and_multi_chunk():
    """V > 32768 spans several vocabulary chunks; g = 1/N (mean loss) via grad_scale."""
    N, V, D = 200, 40000, 64
    H, W, y = synth.random_inputs(N, V, D, seed=41)
    dH, dW = run_backward(H, W, y, None, 1.0 / N)
    ref = oracle.backward(H, W, y, np.float64(np.float32(1.0 / N)), bounds=True)
    compare(dH, ref["dH"], ref["bH"], "dH")
    compare(dW, ref["dW"], ref["bW"], "dW")


def test_backward_matches_torch_autograd_fp32():
    """Against torch autograd on the same bf16 values in fp32 (relative Frobenius)."""
    N, V, D = 384, 5000, 256
    H, W, y = synth.random_inputs(N, V, D, seed=42)
    dH, dW = run_backward(H, W, y, None, 1.0 / N)
    Ht = torch.tensor(synth.bf16_bits_to_f32(H), requires_grad=True)
    Wt = torch.tensor(synth.bf16_bits_to_f32(W), requires_grad=True)
    torch.nn.functional.cross_entropy(Ht @ Wt.T, torch.from_numpy(y)).backward()
    for got, ref in ((dH, Ht.grad.double().numpy()), (dW, Wt.grad.double().numpy())):
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 3e-3


def test_backward_vocab_gradient_sums_to_zero():
    N, V, D = 256, 3000, 128
    H, W, y = synth.random_inputs(N, V, D, seed=43)
    _, dW = run_backward(H, W, y, None, 1.0)
    col = np.abs(dW.sum(axis=0))
    assert col.max() <= 2.0 ** -7 * np.abs(dW).sum(axis=0).max()


def test_backward_deterministic_and_flags_bad_targets():
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 300, 2000, 64
    H, W, y = synth.random_inputs(N, V, D, seed=44)
    Hd, Wd, yd = to_device(H, W, y)
    _, lse, _, _ = flce.forward(Hd, Wd, yd)
    a = [t.clone() for t in flce.backward(Hd, Wd, yd, lse)]
    b = flce.backward(Hd, Wd, yd, lse)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    yb = yd.clone()
    yb[5] = V + 3
    ws = torch.empty(flce.backward_workspace_size(N, V, D), dtype=torch.uint8, device="cuda")
    flce.backward(Hd, Wd, yb, lse, workspace=ws)
    assert flce.check(ws) == flce.ERR_TARGET_OUT_OF_RANGE


# ---------------------------------------------------------------- fp32 inputs
# fp32 H and W: the logits are regenerated from bf16 hi/lo splits (three bf16
# products per fp32 product, about 3 * 2^-16 relative each), dZ is kept as a
# bf16 pair dz + dz_lo (2^-16 relative) and every contraction runs the three
# products hi*hi, hi*lo, lo*hi.  Every entry must meet the bf16 path's bound
# above (2^-8 of the magnitude: a guaranteed bound), and the relative
# Frobenius error must be far below what a bf16 rounding of dZ or of the
# inputs would leave (about 2e-3): under 1e-4.
FP32_FROB = 1e-4


@pytest.mark.parametrize("N,V,D", [(1, 1, 1), (7, 3, 5), (130, 300, 33), (256, 1000, 128),
                                   (64, 20000, 64), (300, 2047, 264)])
def test_backward_fp32_every_element(N, V, D):
    H, W, y = synth.random_inputs(N, V, D, seed=N + 5 * V + 3 * D, dtype="fp32")
    g = np.random.default_rng(N + 1).uniform(-1, 1, N)
    dH, dW = run_backward(H, W, y, g)
    gf = g.astype(np.float32).astype(np.float64)
    ref = oracle.backward(H, W, y, gf, bounds=True)
    for got, r, b, name in ((dH, ref["dH"], ref["bH"], "dH"), (dW, ref["dW"], ref["bW"], "dW")):
        compare(got, r, b, name)
        rel = np.linalg.norm(got - r) / max(np.linalg.norm(r), 1e-30)
        assert rel < FP32_FROB, f"{name}: relative Frobenius error {rel:.2e}"


def test_backward_fp32_mean_loss_multi_chunk_vs_bf16_error():
    """Several vocabulary chunks; and the fp32 path beats the bf16 path on the same values."""
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 200, 40000, 96
    H, W, y = synth.random_inputs(N, V, D, seed=51, dtype="fp32")
    dH, dW = run_backward(H, W, y, None, 1.0 / N)
    ref = oracle.backward(H, W, y, np.float64(np.float32(1.0 / N)), bounds=True)
    e32 = [np.linalg.norm(dH - ref["dH"]) / np.linalg.norm(ref["dH"]),
           np.linalg.norm(dW - ref["dW"]) / np.linalg.norm(ref["dW"])]
    assert max(e32) < FP32_FROB, e32
    # the same fp32 values rounded to bf16 and run on the bf16 path, against their own oracle
    Hb, Wb = synth.round_to_bf16_bits(H), synth.round_to_bf16_bits(W)
    dHb, dWb = run_backward(Hb, Wb, y, None, 1.0 / N)
    refb = oracle.backward(Hb, Wb, y, np.float64(np.float32(1.0 / N)))
    e16 = np.linalg.norm(dHb - refb["dH"]) / np.linalg.norm(refb["dH"])
    assert e32[0] < e16 / 10, (e32, e16)


def test_backward_fp32_deterministic():
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 300, 33000, 40
    H, W, y = synth.random_inputs(N, V, D, seed=52, dtype="fp32")
    Hd, Wd, yd = to_device(H, W, y)
    _, lse, _, _ = flce.forward(Hd, Wd, yd)
    a = [t.clone() for t in flce.backward(Hd, Wd, yd, lse)]
    b = flce.backward(Hd, Wd, yd, lse, check=True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
