"""Edge cases through every Python entry point on the GPU: empty batches, a
one-word vocabulary, and logits in the thousands (the online max must keep
every exponent finite)."""
import math

import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_bf16_b200 import synth
from tests.flce_testing import compare, run, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_cross_entropy_bf16_b200 import build
    build.build()
    oracle.build()


def test_empty_batch_everywhere():
    """N = 0: every entry point returns empty results and launches nothing."""
    import linear_cross_entropy_bf16_b200 as flce
    V, D = 1000, 64
    H = torch.empty(0, D, dtype=torch.bfloat16, device="cuda")
    W = torch.randn(V, D, device="cuda").bfloat16()
    y = torch.empty(0, dtype=torch.int64, device="cuda")
    lse0 = torch.empty(0, device="cuda")
    loss, lse, tgt, mean = flce.forward(H, W, y, check=False)
    assert loss.numel() == lse.numel() == tgt.numel() == 0 and math.isnan(mean.item())
    assert flce.forward_strided(H, W, y.to(torch.int32))[0].numel() == 0
    assert flce.forward(H.float(), W.float(), y)[0].numel() == 0
    dH, dW = flce.backward(H, W, y, lse0)
    assert dH.shape == (0, D) and dW.shape == (V, D) and not dW.abs().any()
    dHs, dWs = flce.backward_shard(H, W[:300].contiguous(), y, lse0, 0, V)
    assert dHs.shape == (0, D) and not dWs.abs().any()
    Wq = torch.zeros(V, D * 4 // 32, dtype=torch.int32, device="cuda")
    sc = torch.ones(V, D // 64, dtype=torch.bfloat16, device="cuda")
    assert flce.forward_quantized(H, Wq, sc, sc, y, 4, 64)[0].numel() == 0
    assert flce.backward_quantized(H, Wq, sc, sc, y, lse0, None, 1.0, 4, 64).shape == (0, D)
    res = flce.forward_host(H.cpu(), W.cpu(), y.cpu())
    assert res[0].numel() == 0
    torch.cuda.synchronize()


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_one_word_vocabulary_gives_zero_loss(dtype):
    """V = 1: lse equals the only logit, so every loss is exactly 0."""
    H, W, _ = synth.random_inputs(300, 1, 128, seed=81, dtype=dtype)
    y = np.zeros(300, dtype=np.int64)
    gpu = run(H, W, y)
    assert np.all(gpu["loss"] == 0.0)
    np.testing.assert_array_equal(gpu["lse"], gpu["target"])
    ref = oracle.forward(H, W, y)
    compare(gpu, ref, mean_ref=None)


@pytest.mark.parametrize("scale", [30.0, 300.0])
def test_logits_in_the_thousands(scale):
    """Rows scaled so logits reach about +-scale * 10 (several thousand at the top
    scale): exp(z - m) stays in range only through the running max."""
    N, V, D = 260, 3000, 128
    H, W, y = synth.random_inputs(N, V, D, seed=82)
    Hs = synth.round_to_bf16_bits(synth.bf16_bits_to_f32(H) * np.float32(scale))
    gpu = run(Hs, W, y)
    ref = oracle.forward(Hs, W, y)
    assert np.abs(ref["max"]).max() > 3 * scale
    assert np.all(np.isfinite(gpu["loss"]))
    # lse and the target logit carry fp32 rounding of values of this size: the
    # 1e-3 bar scales with the logit magnitude here (relative 2^-20 of |max z|)
    tol = np.maximum(1e-3, 2.0 ** -20 * np.abs(ref["max"]))
    for key in ("loss", "lse", "target"):
        assert np.all(np.abs(gpu[key] - ref[key]) <= 2 * tol), key


@pytest.mark.parametrize("N,V,D", [(256, 1 << 20, 128), (65536, 4096, 64), (256, 2048, 16384)])
def test_extreme_extents(N, V, D):
    """A million-word vocabulary (4096 tiles, the 512-slab cap), 65536 tokens, and
    D = 16384: sampled rows against the oracle, properties on every row."""
    import linear_cross_entropy_bf16_b200 as flce
    from tests.flce_testing import check_properties
    H, W, y = synth.random_inputs(N, V, D, seed=N + V + D)
    Hd, Wd, yd = to_device(H, W, y)
    loss, lse, tgt, mean = flce.forward(Hd, Wd, yd, check=True)
    gpu = {"loss": loss.cpu().double().numpy(), "lse": lse.cpu().double().numpy(),
           "target": tgt.cpu().double().numpy(), "mean": float(mean.item())}
    check_properties(gpu, V)
    rows = synth.sample_rows(N, 48, seed=7)
    ref = oracle.forward(H, W, y, rows=rows)
    compare(gpu, ref, rows=rows)
