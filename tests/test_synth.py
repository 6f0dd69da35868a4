"""The seeded input recipe: determinism, bf16 rounding and distributions."""
import math

import numpy as np
import torch

from linear_cross_entropy_bf16_b200 import synth


def test_bf16_rounding_matches_torch_rne():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([1.0, -1.0, 0.0, 1.00390625, 1.01171875, 3.0e38], dtype=np.float32)])
    ours = synth.round_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


def test_generation_is_deterministic_and_chunked():
    a = synth.generate("n1024_v32000_d1024", N=5000, V=9000, D=16)
    b = synth.generate("n1024_v32000_d1024", N=5000, V=9000, D=16)
    for x, z in zip(a, b):
        np.testing.assert_array_equal(x, z)
    H, W, y = a
    assert H.dtype == np.uint16 and W.dtype == np.uint16 and y.dtype == np.int64
    assert H.shape == (5000, 16) and W.shape == (9000, 16) and y.shape == (5000,)
    assert y.min() >= 0 and y.max() < 9000


def test_distributions():
    H, W, y = synth.generate("n1024_v32000_d1024")
    h = synth.bf16_bits_to_f32(H)
    w = synth.bf16_bits_to_f32(W)
    assert abs(h.mean()) < 0.01 and abs(h.std() - 1) < 0.01
    assert abs(w.std() * math.sqrt(1024) - 1) < 0.01
    Ht, Wt, yt = synth.generate("tiny_n256_v2048_d256_fp32")
    assert Ht.dtype == np.float32 and Wt.shape == (2048, 256)


def test_zipf_targets_are_long_tailed():
    y = synth.targets(20000, 128256, 2, "zipf1.1")
    # P(id 0) = 1 / sum_k k^-1.1 over k <= V, about 0.13 here
    p0 = 1.0 / np.sum(np.arange(1, 128257, dtype=np.float64) ** -1.1)
    assert abs((y == 0).mean() - p0) < 0.01
    assert y.max() > 10000


def test_stress_row_scales_span_two_decades():
    s = synth.row_scales(262144, 2048, 4, "row_lognormal_0.1_10") * math.sqrt(2048)
    assert s.min() >= 0.1 * (1 - 1e-6) and s.max() <= 10 * (1 + 1e-6)
    assert s.min() < 0.11 and s.max() > 9.0


def test_sample_rows():
    r = synth.sample_rows(8192, 256, 3)
    assert len(r) == 256 and r[0] == 0 and r[-1] == 8191 and np.all(np.diff(r) > 0)
    np.testing.assert_array_equal(synth.sample_rows(10, 256, 3), np.arange(10))
