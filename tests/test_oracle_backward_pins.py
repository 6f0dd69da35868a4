"""Pins for the oracle's backward (gradients of sum_i g_i loss_i w.r.t. H and W).

Independent checks of the differentiated definition (the page, section 1:
loss_i = logsumexp(Z_i) - Z_{i, y_i}, Z = H W^T): central finite differences
of the oracle's own forward on fp64 inputs, torch autograd on fp64 logits,
exact brute force (rational logits, 50-digit softmax), closed forms and the
zero-sum invariant of the vocabulary gradient.
"""
import math
from fractions import Fraction

import mpmath
import numpy as np
import pytest
import torch

from linear_cross_entropy_bf16_b200 import synth


def f64(a):
    a = np.asarray(a)
    return synth.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def weighted_loss(oracle_mod, H, W, y, g):
    return float(np.dot(oracle_mod.forward(H, W, y)["loss"], g))


def test_finite_differences(oracle_mod):
    rng = np.random.default_rng(30)
    N, V, D = 5, 11, 7
    H = rng.standard_normal((N, D))
    W = rng.standard_normal((V, D)) / 2
    y = rng.integers(0, V, N)
    g = rng.uniform(0.2, 1.5, N)
    out = oracle_mod.backward(H, W, y, g)
    eps = 1e-6
    for (i, k) in [(0, 0), (2, 3), (4, 6), (1, 5)]:
        Hp, Hm = H.copy(), H.copy()
        Hp[i, k] += eps
        Hm[i, k] -= eps
        fd = (weighted_loss(oracle_mod, Hp, W, y, g) - weighted_loss(oracle_mod, Hm, W, y, g)) / (2 * eps)
        assert out["dH"][i, k] == pytest.approx(fd, rel=1e-6, abs=1e-8)
    for (j, k) in [(0, 0), (y[0], 2), (10, 6), (5, 1)]:
        Wp, Wm = W.copy(), W.copy()
        Wp[j, k] += eps
        Wm[j, k] -= eps
        fd = (weighted_loss(oracle_mod, H, Wp, y, g) - weighted_loss(oracle_mod, H, Wm, y, g)) / (2 * eps)
        assert out["dW"][j, k] == pytest.approx(fd, rel=1e-6, abs=1e-8)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_matches_torch_autograd_on_fp64(oracle_mod, dtype):
    rng = np.random.default_rng(31)
    N, V, D = 48, 700, 40
    Hs = rng.standard_normal((N, D)).astype(np.float32)
    Ws = (rng.standard_normal((V, D)) / 6).astype(np.float32)
    H, W = (synth.round_to_bf16_bits(Hs), synth.round_to_bf16_bits(Ws)) if dtype == "bf16" else (Hs, Ws)
    y = rng.integers(0, V, N)
    g = rng.uniform(-1, 1, N)
    out = oracle_mod.backward(H, W, y, g)
    Ht = torch.tensor(f64(H), requires_grad=True)
    Wt = torch.tensor(f64(W), requires_grad=True)
    loss = torch.nn.functional.cross_entropy(Ht @ Wt.T, torch.from_numpy(y), reduction="none")
    (loss * torch.from_numpy(g)).sum().backward()
    np.testing.assert_allclose(out["dH"], Ht.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(out["dW"], Wt.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_brute_force_exact(oracle_mod):
    rng = np.random.default_rng(32)
    N, V, D = 3, 4, 3
    H = synth.round_to_bf16_bits(rng.standard_normal((N, D)).astype(np.float32))
    W = synth.round_to_bf16_bits(rng.standard_normal((V, D)).astype(np.float32))
    y = np.array([0, 3, 1])
    g = np.array([0.5, -1.25, 2.0])
    out = oracle_mod.backward(H, W, y, g, bounds=True)
    Hq = [[Fraction(float(v)) for v in r] for r in f64(H)]
    Wq = [[Fraction(float(v)) for v in r] for r in f64(W)]
    mpmath.mp.dps = 50
    dz = []
    for i in range(N):
        z = [mpmath.mpf(float(sum(Hq[i][k] * Wq[j][k] for k in range(D)))) for j in range(V)]
        lse = mpmath.log(mpmath.fsum(mpmath.e ** v for v in z))
        dz.append([g[i] * (mpmath.e ** (z[j] - lse) - (1 if j == y[i] else 0)) for j in range(V)])
    for i in range(N):
        for k in range(D):
            ref = mpmath.fsum(dz[i][j] * float(Wq[j][k]) for j in range(V))
            mag = mpmath.fsum(abs(dz[i][j]) * abs(float(Wq[j][k])) for j in range(V))
            assert out["dH"][i, k] == pytest.approx(float(ref), rel=1e-12, abs=1e-14)
            assert out["bH"][i, k] == pytest.approx(float(mag), rel=1e-12, abs=1e-14)
    for j in range(V):
        for k in range(D):
            ref = mpmath.fsum(dz[i][j] * float(Hq[i][k]) for i in range(N))
            mag = mpmath.fsum(abs(dz[i][j]) * abs(float(Hq[i][k])) for i in range(N))
            assert out["dW"][j, k] == pytest.approx(float(ref), rel=1e-12, abs=1e-14)
            assert out["bW"][j, k] == pytest.approx(float(mag), rel=1e-12, abs=1e-14)
    for i in range(N):
        row = oracle_mod.grad_logits_row(H, W, y, g[i], i)
        np.testing.assert_allclose(row, [float(v) for v in dz[i]], rtol=1e-12, atol=1e-15)


def test_vocab_gradient_rows_sum_to_zero(oracle_mod):
    """sum_j dL/dZ_ij = g_i (sum_j softmax_ij - 1) = 0, hence sum_j dW_j = 0."""
    H, W, y = synth.random_inputs(60, 500, 24, seed=33)
    g = np.full(60, 1.0 / 60)
    out = oracle_mod.backward(H, W, y, g)
    scale = np.abs(out["dW"]).sum(axis=0).max()
    assert np.abs(out["dW"].sum(axis=0)).max() <= 1e-12 * max(1.0, scale)
    for i in (0, 17, 59):
        assert abs(oracle_mod.grad_logits_row(H, W, y, g[i], i).sum()) <= 1e-15


def test_zero_weights_closed_form(oracle_mod):
    """W = 0: softmax is uniform, so dH = 0 and dW_j = sum_i g_i (1/V - [j == y_i]) H_i."""
    rng = np.random.default_rng(34)
    N, V, D = 9, 13, 5
    H = rng.standard_normal((N, D))
    W = np.zeros((V, D))
    y = rng.integers(0, V, N)
    g = rng.uniform(0.5, 2, N)
    out = oracle_mod.backward(H, W, y, g)
    assert np.all(out["dH"] == 0.0)
    ref = np.zeros((V, D))
    for i in range(N):
        for j in range(V):
            ref[j] += g[i] * (1.0 / V - (1.0 if j == y[i] else 0.0)) * H[i]
    np.testing.assert_allclose(out["dW"], ref, rtol=1e-12, atol=1e-14)


def test_equal_rows_give_zero_dH(oracle_mod):
    """All W rows equal: dH_i = g_i (mean_j W_j - W_{y_i}) = 0."""
    rng = np.random.default_rng(35)
    w = rng.standard_normal(6)
    W = np.tile(w, (20, 1))
    H = rng.standard_normal((4, 6))
    out = oracle_mod.backward(H, W, rng.integers(0, 20, 4), 1.0)
    assert np.abs(out["dH"]).max() <= 1e-14


def test_gradient_is_linear_in_g(oracle_mod):
    H, W, y = synth.random_inputs(30, 200, 16, seed=36)
    rng = np.random.default_rng(37)
    g1, g2 = rng.standard_normal(30), rng.standard_normal(30)
    a = oracle_mod.backward(H, W, y, g1)
    b = oracle_mod.backward(H, W, y, g2)
    c = oracle_mod.backward(H, W, y, 2 * g1 - g2)
    np.testing.assert_allclose(c["dH"], 2 * a["dH"] - b["dH"], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(c["dW"], 2 * a["dW"] - b["dW"], rtol=1e-11, atol=1e-13)


def test_hidden_rows_match_full_backward(oracle_mod):
    H, W, y = synth.random_inputs(40, 300, 24, seed=38)
    g = np.random.default_rng(39).uniform(-1, 1, 40)
    full = oracle_mod.backward(H, W, y, g, bounds=True, want_dW=False)
    rows = np.array([39, 0, 7, 7])
    sub = oracle_mod.grad_hidden_rows(H, W, y, g, rows)
    np.testing.assert_array_equal(sub["dH"], full["dH"][rows])
    np.testing.assert_array_equal(sub["bH"], full["bH"][rows])


# ---------------------------------------------------------------- dW row sampler


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_weight_rows_match_torch_autograd(oracle_mod, dtype):
    """The sampled dW rows against torch autograd on fp64 logits (an independent
    differentiation of the same definition), every element."""
    rng = np.random.default_rng(40)
    N, V, D = 37, 500, 24
    Hs = rng.standard_normal((N, D)).astype(np.float32)
    Ws = (rng.standard_normal((V, D)) / 5).astype(np.float32)
    H, W = (synth.round_to_bf16_bits(Hs), synth.round_to_bf16_bits(Ws)) if dtype == "bf16" else (Hs, Ws)
    y = rng.integers(0, V, N)
    y[:5] = 499                                   # one row that is many tokens' target
    g = rng.uniform(-1, 1, N)
    rows = np.array([499, 0, 250, int(y[7]), 1, 499])
    out = oracle_mod.grad_weight_rows(H, W, y, g, rows)
    Ht = torch.tensor(f64(H))
    Wt = torch.tensor(f64(W), requires_grad=True)
    loss = torch.nn.functional.cross_entropy(Ht @ Wt.T, torch.from_numpy(y), reduction="none")
    (loss * torch.from_numpy(g)).sum().backward()
    np.testing.assert_allclose(out["dW"], Wt.grad.numpy()[rows], rtol=1e-10, atol=1e-13)
    # every token's lse, against the same logits
    lse = torch.logsumexp(Ht @ Wt.detach().T, dim=1).numpy()
    np.testing.assert_allclose(out["lse"], lse, rtol=1e-13, atol=1e-13)


def test_weight_rows_finite_differences(oracle_mod):
    """Central differences of the oracle's own forward on fp64 inputs."""
    rng = np.random.default_rng(41)
    N, V, D = 6, 9, 5
    H = rng.standard_normal((N, D))
    W = rng.standard_normal((V, D)) / 2
    y = rng.integers(0, V, N)
    g = rng.uniform(0.2, 1.5, N)
    rows = np.array([int(y[0]), 8, 3])
    out = oracle_mod.grad_weight_rows(H, W, y, g, rows)
    eps = 1e-6
    for t, j in enumerate(rows):
        for k in range(D):
            Wp, Wm = W.copy(), W.copy()
            Wp[j, k] += eps
            Wm[j, k] -= eps
            fd = (weighted_loss(oracle_mod, H, Wp, y, g) - weighted_loss(oracle_mod, H, Wm, y, g)) / (2 * eps)
            assert out["dW"][t, k] == pytest.approx(fd, rel=1e-6, abs=1e-8)


def test_weight_rows_magnitudes_and_zero_sum(oracle_mod):
    """bW is sum_i |dZ_ij| |H_ik| (exact brute force on a tiny case), and the rows of
    the whole vocabulary sum to zero (sum_j dZ_ij = 0)."""
    rng = np.random.default_rng(42)
    N, V, D = 3, 4, 3
    H = synth.round_to_bf16_bits(rng.standard_normal((N, D)).astype(np.float32))
    W = synth.round_to_bf16_bits(rng.standard_normal((V, D)).astype(np.float32))
    y = np.array([2, 0, 2])
    g = np.array([0.75, -1.5, 1.0])
    out = oracle_mod.grad_weight_rows(H, W, y, g, np.arange(V))
    Hq = [[Fraction(float(v)) for v in r] for r in f64(H)]
    Wq = [[Fraction(float(v)) for v in r] for r in f64(W)]
    mpmath.mp.dps = 50
    dz = []
    for i in range(N):
        z = [mpmath.mpf(float(sum(Hq[i][k] * Wq[j][k] for k in range(D)))) for j in range(V)]
        lse = mpmath.log(mpmath.fsum(mpmath.e ** v for v in z))
        dz.append([g[i] * (mpmath.e ** (z[j] - lse) - (1 if j == y[i] else 0)) for j in range(V)])
    for j in range(V):
        for k in range(D):
            ref = mpmath.fsum(dz[i][j] * float(Hq[i][k]) for i in range(N))
            mag = mpmath.fsum(abs(dz[i][j]) * abs(float(Hq[i][k])) for i in range(N))
            assert out["dW"][j, k] == pytest.approx(float(ref), rel=1e-12, abs=1e-14)
            assert out["bW"][j, k] == pytest.approx(float(mag), rel=1e-12, abs=1e-14)
    H2, W2, y2 = synth.random_inputs(50, 300, 16, seed=43)
    full = oracle_mod.grad_weight_rows(H2, W2, y2, 1.0 / 50, np.arange(300))
    scale = np.abs(full["dW"]).sum(axis=0).max()
    assert np.abs(full["dW"].sum(axis=0)).max() <= 1e-12 * max(1.0, scale)
