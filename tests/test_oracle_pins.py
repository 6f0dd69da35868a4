"""Pins for the fp64 oracle, independent of the oracle itself.

Each check comes from the mathematics of the definition in D. Ineshin,
"Een gefuseerde forward-kernel voor lineaire cross-entropy op Apple-GPU's"
(2026), section 1 (Z = H W^T, loss_i = logsumexp(Z_i) - Z_{i, y_i}):
closed forms, invariants, bounds, a library cross-entropy on fp64 logits, and
exact brute force (rational dot products, 50-digit exp/log).  A dropped term,
a wrong sign or index, or a transposed operand in the oracle fails at least one.
"""
import math
from fractions import Fraction

import mpmath
import numpy as np
import pytest
import torch

from linear_cross_entropy_bf16_b200 import synth


def bf16(x):
    return synth.round_to_bf16_bits(np.asarray(x, dtype=np.float32))


def to_f64(bits_or_f32):
    a = np.asarray(bits_or_f32)
    if a.dtype == np.uint16:
        return synth.bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


# --------------------------------------------------------------------------- closed forms

@pytest.mark.parametrize("V", [1, 2, 7, 1000, 151936])
def test_zero_weights_give_log_V(oracle_mod, V):
    """W = 0: every logit is 0, so lse = ln V and loss = ln V exactly."""
    rng = np.random.default_rng(10)
    N, D = 5, 3
    H = bf16(rng.standard_normal((N, D)))
    W = np.zeros((V, D), dtype=np.uint16)
    y = rng.integers(0, V, N)
    out = oracle_mod.forward(H, W, y)
    assert np.all(out["target"] == 0.0)
    np.testing.assert_allclose(out["lse"], math.log(V), rtol=0, atol=4e-16 * max(1, math.log(V)))
    np.testing.assert_allclose(out["loss"], math.log(V), rtol=0, atol=4e-16 * max(1, math.log(V)))


def test_single_class_gives_zero_loss(oracle_mod):
    """V = 1: lse equals the only logit, so loss = 0 exactly."""
    rng = np.random.default_rng(11)
    H = bf16(rng.standard_normal((6, 16)))
    W = bf16(rng.standard_normal((1, 16)))
    out = oracle_mod.forward(H, W, np.zeros(6, dtype=np.int64))
    assert np.all(out["loss"] == 0.0)
    np.testing.assert_array_equal(out["lse"], out["target"])


def test_equal_logits_give_log_V(oracle_mod):
    """All W rows equal: z_ij = c_i for all j, so lse = c_i + ln V and loss = ln V."""
    rng = np.random.default_rng(12)
    N, V, D = 4, 37, 24
    H = bf16(rng.standard_normal((N, D)))
    w = bf16(rng.standard_normal(D))
    W = np.tile(w, (V, 1))
    y = rng.integers(0, V, N)
    out = oracle_mod.forward(H, W, y)
    c = to_f64(H) @ to_f64(w)
    np.testing.assert_allclose(out["loss"], math.log(V), rtol=1e-14)
    np.testing.assert_allclose(out["lse"], c + math.log(V), rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("V,k,a,b", [(10, 3, 3.0, -2.0), (1000, 1, 8.0, 0.0), (5, 4, -1.5, 0.25)])
def test_two_valued_logits(oracle_mod, V, k, a, b):
    """k columns at logit a, V-k at b: lse = ln(k e^a + (V-k) e^b)."""
    H = bf16([[1.0]])
    W = bf16(np.array([[a]] * k + [[b]] * (V - k)))
    for target, z_t in ((0, a), (V - 1, b)):
        out = oracle_mod.forward(H, W, np.array([target]))
        mpmath.mp.dps = 50
        lse = mpmath.log(k * mpmath.e ** a + (V - k) * mpmath.e ** b)
        # sequential fp64 sum of V terms: relative error of the sum <= (V - 1) u, u = 2^-53
        tol = (V + 2) * 2.0 ** -53 * 2
        assert out["lse"][0] == pytest.approx(float(lse), rel=1e-15, abs=tol)
        assert out["loss"][0] == pytest.approx(float(lse - z_t), rel=1e-15, abs=tol)


@pytest.mark.parametrize("alpha", [2.0, 8.0])
def test_dominant_target_drives_loss_to_zero(oracle_mod, alpha):
    """H_i = alpha W_{y_i}: loss_i = log(1 + sum_{j != y} e^{z_j - z_y}), which -> 0 as alpha grows."""
    rng = np.random.default_rng(13)
    V, D = 50, 16
    W = bf16(np.sign(rng.standard_normal((V, D))))         # +-1 rows: exact in bf16
    y = np.array([3, 17, 49])
    H = bf16(alpha * synth.bf16_bits_to_f32(W[y]))
    out = oracle_mod.forward(H, W, y)
    Z = to_f64(H) @ to_f64(W).T
    mpmath.mp.dps = 50
    for t in range(3):
        zy = Z[t, y[t]]
        tail = mpmath.fsum(mpmath.e ** mpmath.mpf(Z[t, j] - zy) for j in range(V) if j != y[t])
        exact = float(mpmath.log1p(tail))
        # fp64 lse = M + log S carries about one ulp of |z_y| in absolute error
        assert out["loss"][t] == pytest.approx(exact, rel=1e-9, abs=4 * abs(zy) * 2.0 ** -52)
        assert 0.0 <= out["loss"][t] <= exact + 4 * abs(zy) * 2.0 ** -52
    if alpha == 8.0:
        assert np.all(out["loss"] < 1e-12)


# --------------------------------------------------------------------------- invariants

def _small_int_inputs(rng, N, V, D, lo=-4, hi=5):
    H = rng.integers(lo, hi, (N, D)).astype(np.float32)
    W = rng.integers(lo, hi, (V, D)).astype(np.float32) / 8.0
    return bf16(H), bf16(W)


def test_shift_invariance(oracle_mod):
    """Adding one vector c to every W row shifts z_i. by H_i.c: loss unchanged, lse + H_i.c."""
    rng = np.random.default_rng(14)
    N, V, D = 9, 64, 12
    H, W = _small_int_inputs(rng, N, V, D)
    c = rng.integers(-3, 4, D).astype(np.float32) / 4.0
    W2 = bf16(synth.bf16_bits_to_f32(W) + c)                 # exact: small dyadic values
    assert np.array_equal(to_f64(W2), to_f64(W) + c)
    y = rng.integers(0, V, N)
    a = oracle_mod.forward(H, W, y)
    b = oracle_mod.forward(H, W2, y)
    shift = to_f64(H) @ c.astype(np.float64)
    np.testing.assert_allclose(b["loss"], a["loss"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(b["lse"], a["lse"] + shift, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(b["target"], a["target"] + shift, rtol=0, atol=1e-12)


def test_vocab_permutation_invariance(oracle_mod):
    """Permuting W rows together with the target ids leaves every output unchanged."""
    rng = np.random.default_rng(15)
    N, V, D = 7, 300, 20
    H = bf16(rng.standard_normal((N, D)))
    W = bf16(rng.standard_normal((V, D)) / math.sqrt(D))
    y = rng.integers(0, V, N)
    perm = rng.permutation(V)            # new row r holds old row perm[r]
    inv = np.argsort(perm)
    a = oracle_mod.forward(H, W, y)
    b = oracle_mod.forward(H, W[perm], inv[y])
    np.testing.assert_array_equal(b["target"], a["target"])
    np.testing.assert_allclose(b["lse"], a["lse"], rtol=1e-14)
    np.testing.assert_allclose(b["loss"], a["loss"], rtol=1e-12, atol=1e-14)


def test_row_permutation_equivariance(oracle_mod):
    rng = np.random.default_rng(16)
    N, V, D = 11, 40, 8
    H = bf16(rng.standard_normal((N, D)))
    W = bf16(rng.standard_normal((V, D)))
    y = rng.integers(0, V, N)
    perm = rng.permutation(N)
    a = oracle_mod.forward(H, W, y)
    b = oracle_mod.forward(H[perm], W, y[perm])
    for k in ("loss", "lse", "target"):
        np.testing.assert_array_equal(b[k], a[k][perm])


def test_bounds(oracle_mod):
    """max_j z_ij <= lse_i <= max_j z_ij + ln V, and loss_i >= 0."""
    rng = np.random.default_rng(17)
    N, V, D = 16, 500, 32
    H = bf16(rng.standard_normal((N, D)) * 3)
    W = bf16(rng.standard_normal((V, D)))
    y = rng.integers(0, V, N)
    out = oracle_mod.forward(H, W, y)
    Z = to_f64(H) @ to_f64(W).T
    zmax = Z.max(axis=1)
    np.testing.assert_allclose(out["max"], zmax, rtol=1e-13)
    assert np.all(out["lse"] >= out["max"])
    assert np.all(out["lse"] <= out["max"] + math.log(V) * (1 + 1e-15))
    assert np.all(out["loss"] >= 0.0)


# --------------------------------------------------------------------------- library and brute force

@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_matches_torch_cross_entropy_on_fp64_logits(oracle_mod, dtype):
    """The library special case: F.cross_entropy on fp64 logits H W^T."""
    rng = np.random.default_rng(18)
    N, V, D = 64, 1000, 64
    Hs = rng.standard_normal((N, D)).astype(np.float32)
    Ws = (rng.standard_normal((V, D)) / 8).astype(np.float32)
    H, W = (bf16(Hs), bf16(Ws)) if dtype == "bf16" else (Hs, Ws)
    y = rng.integers(0, V, N)
    out = oracle_mod.forward(H, W, y)
    Z = torch.from_numpy(to_f64(H)) @ torch.from_numpy(to_f64(W)).T
    ref = torch.nn.functional.cross_entropy(Z, torch.from_numpy(y), reduction="none").numpy()
    np.testing.assert_allclose(out["loss"], ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out["lse"], torch.logsumexp(Z, dim=1).numpy(), rtol=1e-12)
    np.testing.assert_allclose(out["target"], Z[np.arange(N), y].numpy(), rtol=1e-12, atol=1e-12)
    ref_mean = torch.nn.functional.cross_entropy(Z, torch.from_numpy(y), reduction="mean").item()
    assert oracle_mod.mean(out["loss"]) == pytest.approx(ref_mean, rel=1e-13)


def test_logits_row_orientation(oracle_mod):
    """z_ij pairs row i of H with row j of W (not a transposed operand)."""
    rng = np.random.default_rng(19)
    N, V, D = 3, 5, 4
    H = bf16(rng.integers(-3, 4, (N, D)))
    W = bf16(rng.integers(-3, 4, (V, D)))
    Hf, Wf = to_f64(H), to_f64(W)
    for i in range(N):
        z = oracle_mod.logits_row(H, W, i)
        assert [float(v) for v in z] == [float(sum(Hf[i, k] * Wf[j, k] for k in range(D))) for j in range(V)]


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_brute_force_exact(oracle_mod, seed, dtype):
    """N, V, D <= 8: rational dot products and 50-digit exp/log."""
    rng = np.random.default_rng(100 + seed)
    N, V, D = (int(v) for v in rng.integers(1, 9, 3))
    Hs = (rng.standard_normal((N, D)) * 2).astype(np.float32)
    Ws = (rng.standard_normal((V, D)) * 2).astype(np.float32)
    H, W = (bf16(Hs), bf16(Ws)) if dtype == "bf16" else (Hs, Ws)
    y = rng.integers(0, V, N)
    out = oracle_mod.forward(H, W, y)
    Hq = [[Fraction(float(v)) for v in row] for row in to_f64(H)]
    Wq = [[Fraction(float(v)) for v in row] for row in to_f64(W)]
    mpmath.mp.dps = 50
    losses = []
    for i in range(N):
        z = [sum((Hq[i][k] * Wq[j][k] for k in range(D)), Fraction(0)) for j in range(V)]
        zm = [mpmath.mpf(q.numerator) / q.denominator for q in z]
        lse = mpmath.log(mpmath.fsum(mpmath.e ** v for v in zm))
        loss = lse - zm[y[i]]
        losses.append(loss)
        assert out["target"][i] == pytest.approx(float(zm[y[i]]), rel=1e-15, abs=1e-15)
        assert out["lse"][i] == pytest.approx(float(lse), rel=1e-14, abs=1e-14)
        assert out["loss"][i] == pytest.approx(float(loss), rel=1e-13, abs=1e-13)
    assert oracle_mod.mean(out["loss"]) == pytest.approx(float(mpmath.fsum(losses) / N), rel=1e-13, abs=1e-14)


def test_row_subset_matches_full(oracle_mod):
    rng = np.random.default_rng(20)
    H, W, y = synth.random_inputs(40, 333, 24, seed=7)
    full = oracle_mod.forward(H, W, y)
    rows = np.array([39, 0, 17, 17, 5])
    sub = oracle_mod.forward(H, W, y, rows=rows)
    for k in full:
        np.testing.assert_array_equal(sub[k], full[k][rows])


def test_mean_is_plain_average(oracle_mod):
    rng = np.random.default_rng(21)
    x = rng.uniform(0, 20, 1001)
    assert oracle_mod.mean(x) == pytest.approx(math.fsum(x) / len(x), rel=1e-15)
    assert math.isnan(oracle_mod.mean(np.zeros(0)))


def test_invalid_target_raises(oracle_mod):
    H, W, y = synth.random_inputs(4, 10, 8, seed=1)
    for bad in (-1, 10):
        yb = y.copy()
        yb[2] = bad
        with pytest.raises(oracle_mod.OracleError):
            oracle_mod.forward(H, W, yb)


def test_stress_scale_logits_are_finite(oracle_mod):
    """Logit std up to ~10 (the stress recipe): the two-pass lse stays finite and exact."""
    H, W, y = synth.generate("stress_n16384_v262144_d2048", N=4, V=3000, D=64)
    out = oracle_mod.forward(H, W, y)
    Z = torch.from_numpy(to_f64(H)) @ torch.from_numpy(to_f64(W)).T
    ref = torch.nn.functional.cross_entropy(Z, torch.from_numpy(y), reduction="none").numpy()
    assert np.all(np.isfinite(out["loss"]))
    np.testing.assert_allclose(out["loss"], ref, rtol=1e-12, atol=1e-12)
