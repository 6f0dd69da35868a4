"""Pins of the oracle's quantised-head forward (CPU only).

The page (section 2) says its MLX prototype supported dense and quantised
output heads but does not define the quantised format.  Reading taken here:
MLX's affine group quantisation, W_jk = s_{j, k // G} * q_jk + b_{j, k // G},
with `bits`-bit codes packed 32 / bits per uint32, lowest bits first.  These
tests pin the oracle's unpacking and dequantisation to that reading with
literal words, to an independent encoder on exactly representable weights,
to closed forms, and to the dense oracle (itself pinned elsewhere).
"""
import math

import numpy as np
import pytest

import oracle
from linear_cross_entropy_bf16_b200 import synth


def bf16(x):
    return synth.round_to_bf16_bits(np.asarray(x, dtype=np.float32))


def ones_groups(V, D, G, value=1.0):
    return np.full((V, D // G), bf16(value), dtype=np.uint16)


@pytest.mark.parametrize("bits,word,codes", [
    (4, 0x76543210, [0, 1, 2, 3, 4, 5, 6, 7]),
    (4, 0xF0E1D2C3, [3, 12, 2, 13, 1, 14, 0, 15]),
    (8, 0x04030201, [1, 2, 3, 4]),
    (8, 0xFF00807F, [127, 128, 0, 255]),
    (2, 0xE4E4E4E4, [0, 1, 2, 3] * 4),
    (2, 0x0000001B, [3, 2, 1, 0] + [0] * 12),
])
def test_packing_literal_words(bits, word, codes):
    """Element k of a row sits at bit offset bits * (k mod (32/bits)), lowest bits first."""
    per = 32 // bits
    G = 32
    D = G                                 # one group; the word repeats across the row
    words = D // per
    wq = np.full((1, words), word, dtype=np.uint32)
    W = oracle.dequantize(wq, ones_groups(1, D, G), ones_groups(1, D, G, 0.0), bits, G)
    assert W.shape == (1, D)
    np.testing.assert_array_equal(W[0, :per], np.array(codes, dtype=np.float64))
    np.testing.assert_array_equal(W[0], np.tile(np.array(codes, dtype=np.float64), words))


def test_scale_and_bias_per_group_and_row():
    """Distinct scales and biases per (row, group) land on the right elements."""
    V, D, G, bits = 3, 64, 32, 4
    q = (np.arange(V * D).reshape(V, D) * 7 + 3) % 16
    s = np.array([[0.5, 2.0], [0.25, 4.0], [1.0, 0.125]], dtype=np.float32)
    b = np.array([[-3.0, 1.0], [0.5, -8.0], [0.0, 16.0]], dtype=np.float32)
    W = oracle.dequantize(synth.pack_codes(q, bits), bf16(s), bf16(b), bits, G)
    for j in range(V):
        for k in range(D):
            g = k // G
            assert W[j, k] == float(s[j, g]) * float(q[j, k]) + float(b[j, g]), (j, k)


@pytest.mark.parametrize("bits,G", [(4, 64), (2, 32), (8, 128), (4, 32)])
def test_exact_weights_reduce_to_dense_oracle(bits, G):
    """W chosen on the quantisation grid (power-of-two scales, small integer biases)
    is exact in bf16, so the quantised forward must equal the dense one exactly."""
    rng = np.random.default_rng(bits * 100 + G)
    V, D, N = 37, 2 * G if G < 128 else G, 9
    # codes below 128 keep s * q + b within bf16's 8 significant bits for 8-bit codes
    levels = min(2 ** bits, 128)
    q = rng.integers(0, levels, (V, D))
    s = 2.0 ** rng.integers(-6, -2, (V, D // G))
    b = rng.integers(-4, 5, (V, D // G)).astype(np.float64) / 8
    Wexact = s.repeat(G, axis=1) * q + b.repeat(G, axis=1)
    # pack with Python ints, independent of synth.pack_codes
    per = 32 // bits
    words = np.zeros((V, D // per), dtype=np.uint32)
    for j in range(V):
        for w in range(D // per):
            acc = 0
            for t in range(per):
                acc |= int(q[j, w * per + t]) << (bits * t)
            words[j, w] = acc
    Wd = oracle.dequantize(words, bf16(s), bf16(b), bits, G)
    np.testing.assert_array_equal(Wd, Wexact)
    Wb = bf16(Wexact)
    assert np.array_equal(synth.bf16_bits_to_f32(Wb).astype(np.float64), Wexact)   # exact in bf16
    H = synth.round_to_bf16_bits(rng.standard_normal((N, D)).astype(np.float32))
    y = rng.integers(0, V, N)
    dense = oracle.forward(H, Wb, y)
    quant = oracle.forward_quantized(H, words, bf16(s), bf16(b), y, bits, G)
    for key in ("loss", "lse", "target", "max"):
        np.testing.assert_array_equal(quant[key], dense[key])


def test_zero_scale_and_bias_give_log_V():
    V, D, G, N = 50, 64, 64, 4
    H = synth.round_to_bf16_bits(np.random.default_rng(1).standard_normal((N, D)).astype(np.float32))
    wq = np.full((V, D // 8), 0xFFFFFFFF, dtype=np.uint32)
    zeros = ones_groups(V, D, G, 0.0)
    out = oracle.forward_quantized(H, wq, zeros, zeros, np.arange(N), 4, G)
    np.testing.assert_allclose(out["loss"], math.log(V), rtol=0, atol=1e-12)


def test_bias_only_closed_form():
    """s = 0: W_jk = b_{j,g}; with H = 1 every logit is z_j = G * sum_g b_jg."""
    V, D, G, N = 6, 128, 32, 3
    b = (np.arange(V * (D // G)).reshape(V, D // G) % 5 - 2).astype(np.float32) / 4
    H = np.full((N, D), bf16(1.0), dtype=np.uint16)
    wq = np.random.default_rng(2).integers(0, 2 ** 32, (V, D // 8), dtype=np.uint64).astype(np.uint32)
    out = oracle.forward_quantized(H, wq, ones_groups(V, D, G, 0.0), bf16(b), np.array([0, 3, 5]), 4, G)
    z = [G * math.fsum(float(v) for v in b[j]) for j in range(V)]
    m = max(z)
    lse = m + math.log(math.fsum(math.exp(v - m) for v in z))
    np.testing.assert_allclose(out["lse"], lse, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["loss"], [lse - z[0], lse - z[3], lse - z[5]], rtol=0, atol=1e-12)


def test_rows_subset_matches_full():
    H, (wq, s, b), y = synth.generate_quantized("n1024_v32000_d1024", 4, 64, N=20, V=300, D=128)
    full = oracle.forward_quantized(H, wq, s, b, y, 4, 64)
    rows = np.array([19, 0, 7])
    sub = oracle.forward_quantized(H, wq, s, b, y, 4, 64, rows=rows)
    for key in ("loss", "lse", "target"):
        np.testing.assert_array_equal(sub[key], full[key][rows])


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_synth_quantizer_round_trip_bound(bits):
    """The input quantiser and the oracle's dequantiser agree: every weight comes back
    within half a step, plus what bf16 rounding of the scale (over 2^bits - 1 steps)
    and of the bias can add."""
    rng = np.random.default_rng(bits)
    W = rng.standard_normal((200, 256)).astype(np.float32) / 16
    G = 64
    wq, s, b = synth.quantize_affine(W, bits, G)
    Wd = oracle.dequantize(wq, s, b, bits, G)
    sc = synth.bf16_bits_to_f32(s).astype(np.float64).repeat(G, axis=1)
    bb = np.abs(synth.bf16_bits_to_f32(b).astype(np.float64)).repeat(G, axis=1)
    bound = (0.5 + (2 ** bits - 1) * 2.0 ** -8) * sc + 2.0 ** -7 * bb
    assert np.all(np.abs(Wd - W) <= bound)


def test_rejects_bad_formats():
    H = np.zeros((2, 64), dtype=np.uint16)
    wq = np.zeros((3, 24), dtype=np.uint32)       # 3 bits is not supported
    s = np.zeros((3, 1), dtype=np.uint16)
    with pytest.raises((oracle.OracleError, ValueError)):
        oracle.forward_quantized(H, wq, s, s, np.zeros(2, dtype=np.int64), 3, 64)
    with pytest.raises(oracle.OracleError):          # group size 16 is not supported
        oracle.dequantize(np.zeros((3, 8), dtype=np.uint32), np.zeros((3, 4), dtype=np.uint16),
                          np.zeros((3, 4), dtype=np.uint16), 4, 16)
    with pytest.raises(oracle.OracleError):          # target out of range
        oracle.forward_quantized(H, np.zeros((3, 8), dtype=np.uint32), s, s,
                                 np.array([0, 3]), 4, 64)
