"""GPU parity of the quantised-head forward (flce_forward_quantized) against the oracle.

The head is MLX's affine group format, W = s * q + b per group of G along D
(the page's section 2 mentions quantised heads without a format; this is the
reading the library and the oracle both take).  The GPU expands W to bf16
[hi | lo] and forms H hi^T + H lo^T per K block: per weight |W - hi - lo| <=
2^-16 |W|, so the bar is the forward's: |d loss|, |d lse| <= 1e-3 per token,
|d mean| / |mean| <= 1e-5.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_bf16_b200 import synth
from tests.flce_testing import check_properties, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_cross_entropy_bf16_b200 import build
    build.build()
    oracle.build()


def to_dev(H, wq, s, b, y):
    dev = torch.device("cuda:0")
    Hd = torch.from_numpy(np.ascontiguousarray(H)).view(torch.bfloat16).to(dev)
    wqd = torch.from_numpy(np.ascontiguousarray(wq).view(np.int32)).to(dev)
    sd = torch.from_numpy(np.ascontiguousarray(s)).view(torch.bfloat16).to(dev)
    bd = torch.from_numpy(np.ascontiguousarray(b)).view(torch.bfloat16).to(dev)
    yd = torch.from_numpy(np.ascontiguousarray(y, dtype=np.int64)).to(dev)
    return Hd, wqd, sd, bd, yd


def run_q(H, wq, s, b, y, bits, G, check=True):
    import linear_cross_entropy_bf16_b200 as flce
    loss, lse, tgt, mean = flce.forward_quantized(*to_dev(H, wq, s, b, y), bits, G, check=check)
    torch.cuda.synchronize()
    return {"loss": loss.cpu().double().numpy(), "lse": lse.cpu().double().numpy(),
            "target": tgt.cpu().double().numpy(), "mean": float(mean.item())}


def inputs(N, V, D, bits, G, seed, w_std=None):
    H, Wf, y = synth.random_inputs(N, V, D, seed=seed, dtype="fp32", w_std=w_std)
    H = synth.round_to_bf16_bits(H)
    return (H,) + synth.quantize_affine(Wf, bits, G) + (y,)


SHAPES = [
    # N, V, D, bits, G
    (1, 1, 64, 4, 64), (7, 300, 64, 4, 32), (129, 2047, 128, 4, 64), (300, 1000, 256, 2, 128),
    (513, 3000, 192, 8, 64), (200, 5000, 96, 4, 32), (64, 40000, 64, 4, 64),
    (257, 16389, 128, 8, 32), (130, 900, 320, 2, 64),
]


@pytest.mark.parametrize("N,V,D,bits,G", SHAPES)
def test_quantized_shapes_every_row(N, V, D, bits, G):
    """Ragged N and V, a padded K segment (D % 64 != 0), several 16384-row chunks with a
    ragged last one (V = 40000, V = 16389), all code widths and group sizes."""
    H, wq, s, b, y = inputs(N, V, D, bits, G, seed=N + V + D + bits)
    gpu = run_q(H, wq, s, b, y, bits, G)
    ref = oracle.forward_quantized(H, wq, s, b, y, bits, G)
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))


@pytest.mark.parametrize("where", [0, 16383, 16384, 32767, 32768, 39999])
def test_quantized_targets_at_chunk_edges(where):
    N, V, D, bits, G = 300, 40000, 64, 4, 64
    H, wq, s, b, _ = inputs(N, V, D, bits, G, seed=11)
    y = np.full(N, where, dtype=np.int64)
    y[::3] = np.random.default_rng(where).integers(0, V, len(y[::3]))
    gpu = run_q(H, wq, s, b, y, bits, G)
    ref = oracle.forward_quantized(H, wq, s, b, y, bits, G)
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))


def test_quantized_matches_dense_on_exact_weights():
    """Weights on the grid and exact in bf16: the quantised path (lo parts all zero)
    and the dense bf16 path see the same W."""
    import linear_cross_entropy_bf16_b200 as flce
    rng = np.random.default_rng(5)
    N, V, D, G, bits = 400, 3000, 128, 64, 4
    q = rng.integers(0, 16, (V, D))
    sc = 2.0 ** rng.integers(-7, -4, (V, D // G))
    bi = rng.integers(-4, 5, (V, D // G)) / 64.0
    W = sc.repeat(G, axis=1) * q + bi.repeat(G, axis=1)
    Wb = synth.round_to_bf16_bits(W.astype(np.float32))
    assert np.array_equal(synth.bf16_bits_to_f32(Wb).astype(np.float64), W)
    H = synth.round_to_bf16_bits(rng.standard_normal((N, D)).astype(np.float32))
    y = rng.integers(0, V, N)
    s16 = synth.round_to_bf16_bits(sc.astype(np.float32))
    b16 = synth.round_to_bf16_bits(bi.astype(np.float32))
    gq = run_q(H, synth.pack_codes(q, bits), s16, b16, y, bits, G)
    Hd, _, _, _, yd = to_dev(H, np.zeros((1, 1), np.uint32), s16, b16, y)
    Wd = torch.from_numpy(Wb).view(torch.bfloat16).cuda()
    loss, lse, tgt, mean = flce.forward(Hd, Wd, yd, check=True)
    np.testing.assert_allclose(gq["target"], tgt.cpu().double().numpy(), rtol=0, atol=1e-5)
    np.testing.assert_allclose(gq["lse"], lse.cpu().double().numpy(), rtol=0, atol=1e-5)


def test_quantized_deterministic_and_target_check():
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D, bits, G = 300, 20000, 128, 4, 64
    H, wq, s, b, y = inputs(N, V, D, bits, G, seed=3)
    args = to_dev(H, wq, s, b, y)
    first = flce.forward_quantized(*args, bits, G, check=True)
    second = flce.forward_quantized(*args, bits, G, check=True)
    for a, c in zip(first, second):
        assert torch.equal(a, c)
    y_bad = args[4].clone()
    y_bad[17] = V
    loss = flce.forward_quantized(*args[:4], y_bad, bits, G)[0]
    torch.cuda.synchronize()
    assert torch.isnan(loss[17]) and torch.isfinite(loss[:17]).all()
    with pytest.raises(flce.FlceError):
        flce.forward_quantized(*args[:4], y_bad, bits, G, check=True)


def test_quantized_page_shape_sampled_rows():
    """N=8192 V=151936 D=4096 with W quantised to 4 bits in groups of 64: 10 chunks, the
    last one ragged; sampled rows against the oracle, properties on every row."""
    N, V, D, bits, G = 8192, 151936, 4096, 4, 64
    H, (wq, s, b), y = synth.generate_quantized(synth.HEADLINE, bits, G)
    gpu = run_q(H, wq, s, b, y, bits, G)
    check_properties(gpu, V)
    rows = synth.sample_rows(N, 24, seed=41)
    ref = oracle.forward_quantized(H, wq, s, b, y, bits, G, rows=rows)
    compare(gpu, ref, rows=rows)
    # logits of a 4-bit head of N(0, 1/D) weights are still about N(0, 1): loss near ln V + 1/2
    assert abs(gpu["mean"] - (math.log(V) + 0.5)) < 0.2


# ---------------------------------------------------------------- backward (dH only)
# dZ is rounded to bf16 before dH = dZ (W_hi + W_lo) is accumulated in fp32,
# so |d dH_ik| <= 2^-8 sum_j |dZ_ij| |W_jk| (the oracle's bH on the
# dequantised W; the hi/lo split adds only 2^-16 of it), plus a tiny floor.


def run_q_backward(H, wq, s, b, y, bits, G, g=None, scale=1.0):
    import linear_cross_entropy_bf16_b200 as flce
    Hd, wqd, sd, bd, yd = to_dev(H, wq, s, b, y)
    _, lse, _, _ = flce.forward_quantized(Hd, wqd, sd, bd, yd, bits, G, check=True)
    gd = torch.from_numpy(np.asarray(g, dtype=np.float32)).cuda() if g is not None else None
    dH = flce.backward_quantized(Hd, wqd, sd, bd, yd, lse, gd, scale, bits, G, check=True)
    torch.cuda.synchronize()
    return dH.cpu().double().numpy()


@pytest.mark.parametrize("N,V,D,bits,G", [(1, 1, 64, 4, 64), (7, 300, 64, 4, 32),
                                          (130, 2047, 128, 4, 64), (300, 5000, 96, 2, 32),
                                          (200, 40000, 64, 8, 64), (257, 32773, 192, 4, 64)])
def test_quantized_backward_every_element(N, V, D, bits, G):
    H, wq, s, b, y = inputs(N, V, D, bits, G, seed=3 * N + V + D)
    g = np.random.default_rng(N).uniform(-1, 1, N)
    dH = run_q_backward(H, wq, s, b, y, bits, G, g)
    Wd = oracle.dequantize(wq, s, b, bits, G)
    Hf = synth.bf16_bits_to_f32(H).astype(np.float64)
    ref = oracle.backward(Hf, Wd, y, g.astype(np.float32).astype(np.float64), bounds=True)
    err = np.abs(dH - ref["dH"])
    lim = 2.0 ** -8 * ref["bH"] + 1e-7
    worst = np.unravel_index(np.argmax(err - lim), err.shape)
    assert np.all(err <= lim), (worst, err[worst], lim[worst])
    assert np.linalg.norm(dH - ref["dH"]) / max(np.linalg.norm(ref["dH"]), 1e-30) < 3e-3


def test_quantized_backward_deterministic_and_target_check():
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D, bits, G = 300, 36000, 128, 4, 64
    H, wq, s, b, y = inputs(N, V, D, bits, G, seed=9)
    Hd, wqd, sd, bd, yd = to_dev(H, wq, s, b, y)
    _, lse, _, _ = flce.forward_quantized(Hd, wqd, sd, bd, yd, bits, G)
    a = flce.backward_quantized(Hd, wqd, sd, bd, yd, lse, None, 1.0 / N, bits, G).clone()
    c = flce.backward_quantized(Hd, wqd, sd, bd, yd, lse, None, 1.0 / N, bits, G, check=True)
    assert torch.equal(a, c)
    yb = yd.clone()
    yb[3] = -1
    with pytest.raises(flce.FlceError):
        flce.backward_quantized(Hd, wqd, sd, bd, yb, lse, None, 1.0, bits, G, check=True)
