"""Seeded synthetic inputs for the fused linear cross-entropy forward.

This module holds the input recipe only: shapes, distributions, seeds and the
rounding of fp32 samples to bf16.  It contains none of the loss arithmetic, so
both the CUDA path and the CPU oracle can be fed from it.

Recipe (all on the host, numpy ``default_rng``):
  * H (N, D): standard normal fp32.
  * W (V, D): standard normal fp32 times 1/sqrt(D), so each logit is about
    N(0, 1).  For the stress workload row j is scaled instead by
    sigma_j = exp(U(ln 0.1, ln 10)) / sqrt(D), which spreads logit scales over
    two decades and exercises the online-max rescaling.
  * y (N,): uniform in [0, V) or a finite Zipf law P(id = k) ~ (k + 1)^-1.1.
  * bf16 workloads round the fp32 samples to bf16 with round-to-nearest-even;
    the oracle and the GPU both read those exact bit patterns.
Large matrices are generated in row chunks of ``CHUNK_ROWS`` with one
independent generator per chunk, seeded by (seed, stream, chunk), so the bytes
do not depend on how many threads fill them.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

CHUNK_ROWS = 4096

# generator stream ids inside one workload seed
_S_H, _S_W, _S_SIGMA, _S_Y, _S_ROWS = 1, 2, 3, 4, 5


@dataclass(frozen=True)
class Workload:
    name: str
    N: int
    V: int
    D: int
    dtype: str          # "bf16" or "fp32" (storage and compute input type)
    targets: str        # "uniform" or "zipf1.1"
    w_scale: str        # "inv_sqrt_d" or "row_lognormal_0.1_10"
    seed: int

    @property
    def flops(self) -> int:
        """Dense contraction work of one forward: 2 N V D."""
        return 2 * self.N * self.V * self.D


# The five workloads the forward is checked and measured on.
WORKLOADS = {
    w.name: w for w in (
        Workload("tiny_n256_v2048_d256_fp32", 256, 2048, 256, "fp32", "uniform", "inv_sqrt_d", 0),
        Workload("n1024_v32000_d1024", 1024, 32000, 1024, "bf16", "uniform", "inv_sqrt_d", 1),
        Workload("n4096_v128256_d4096_zipf", 4096, 128256, 4096, "bf16", "zipf1.1", "inv_sqrt_d", 2),
        Workload("n8192_v151936_d4096", 8192, 151936, 4096, "bf16", "uniform", "inv_sqrt_d", 3),
        Workload("stress_n16384_v262144_d2048", 16384, 262144, 2048, "bf16", "zipf1.1",
                 "row_lognormal_0.1_10", 4),
    )
}
# The production shape from the page (N=8192, V=151936, D=4096): the headline workload.
HEADLINE = "n8192_v151936_d4096"


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest, ties to even.

    Inputs are finite (normal samples), so no NaN handling is needed.
    """
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _threads() -> int:
    try:
        return max(1, min(32, len(os.sched_getaffinity(0))))
    except AttributeError:  # pragma: no cover
        return max(1, min(32, os.cpu_count() or 1))


def _fill_rows(rows: int, cols: int, seed: int, stream: int, dtype: str, row_scale) -> np.ndarray:
    out = np.empty((rows, cols), dtype=np.uint16 if dtype == "bf16" else np.float32)

    def work(c):
        r0 = c * CHUNK_ROWS
        r1 = min(rows, r0 + CHUNK_ROWS)
        rng = np.random.default_rng([seed, stream, c])
        x = rng.standard_normal((r1 - r0, cols), dtype=np.float32)
        if row_scale is not None:
            x *= row_scale[r0:r1, None]
        if dtype == "bf16":
            out[r0:r1] = round_to_bf16_bits(x)
        else:
            out[r0:r1] = x

    nchunks = (rows + CHUNK_ROWS - 1) // CHUNK_ROWS
    if nchunks <= 1:
        for c in range(nchunks):
            work(c)
    else:
        with ThreadPoolExecutor(min(_threads(), nchunks)) as ex:
            list(ex.map(work, range(nchunks)))
    return out


def row_scales(V: int, D: int, seed: int, w_scale: str) -> np.ndarray:
    if w_scale == "inv_sqrt_d":
        return np.full(V, 1.0 / math.sqrt(D), dtype=np.float32)
    if w_scale == "row_lognormal_0.1_10":
        rng = np.random.default_rng([seed, _S_SIGMA])
        u = rng.uniform(math.log(0.1), math.log(10.0), V)
        return (np.exp(u) / math.sqrt(D)).astype(np.float32)
    raise ValueError(w_scale)


def targets(N: int, V: int, seed: int, kind: str) -> np.ndarray:
    rng = np.random.default_rng([seed, _S_Y])
    if kind == "uniform":
        return rng.integers(0, V, N, dtype=np.int64)
    if kind == "zipf1.1":
        p = np.arange(1, V + 1, dtype=np.float64) ** -1.1
        p /= p.sum()
        return rng.choice(V, N, p=p).astype(np.int64)
    raise ValueError(kind)


def generate(w: Workload | str, N: int | None = None, V: int | None = None,
             D: int | None = None, token_stream: int = 0):
    """Return (H, W, y) numpy arrays for workload ``w`` (optionally reshaped).

    H and W are uint16 bf16 bit patterns for bf16 workloads, float32 otherwise.
    ``token_stream`` > 0 draws a different, equally distributed batch of tokens
    and targets (one per data-parallel rank) against the same W.
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    N = w.N if N is None else N
    V = w.V if V is None else V
    D = w.D if D is None else D
    tseed = w.seed if token_stream == 0 else w.seed * 1000003 + token_stream
    H = _fill_rows(N, D, tseed, _S_H, w.dtype, None)
    W = _fill_rows(V, D, w.seed, _S_W, w.dtype, row_scales(V, D, w.seed, w.w_scale))
    y = targets(N, V, tseed, w.targets)
    return H, W, y


def random_inputs(N: int, V: int, D: int, seed: int, dtype: str = "bf16",
                  w_std: float | None = None, targets_kind: str = "uniform"):
    """Small seeded inputs of any shape (tests): H ~ N(0,1), W ~ N(0, w_std^2)."""
    std = (1.0 / math.sqrt(D)) if w_std is None else w_std
    H = _fill_rows(N, D, seed, _S_H, dtype, None)
    W = _fill_rows(V, D, seed, _S_W, dtype, np.full(V, std, dtype=np.float32))
    y = targets(N, V, seed, targets_kind)
    return H, W, y


def sample_rows(N: int, k: int, seed: int) -> np.ndarray:
    """A seeded sorted subset of k row indices that always holds the first and last row."""
    if k >= N:
        return np.arange(N, dtype=np.int64)
    rng = np.random.default_rng([seed, _S_ROWS])
    inner = rng.choice(np.arange(1, N - 1), size=max(0, k - 2), replace=False)
    return np.sort(np.concatenate([[0, N - 1], inner]).astype(np.int64))


# ---------------------------------------------------------------- quantised heads

def pack_codes(q: np.ndarray, bits: int) -> np.ndarray:
    """Pack unsigned `bits`-bit codes (V, D) into uint32 words (V, D * bits / 32),
    32 / bits codes per word, element k at bit offset bits * (k mod (32 / bits))."""
    per = 32 // bits
    V, D = q.shape
    q = q.astype(np.uint32).reshape(V, D // per, per)
    shifts = (np.arange(per, dtype=np.uint32) * bits)[None, None, :]
    return np.bitwise_or.reduce(q << shifts, axis=2).astype(np.uint32)


def quantize_affine(W: np.ndarray, bits: int = 4, group_size: int = 64):
    """Affine group quantisation of an fp32 (V, D) matrix, MLX-style: per group of
    `group_size` elements along D, bias = bf16(min), scale = bf16((max - min) / (2^bits - 1))
    and q = clip(round((w - bias) / scale), 0, 2^bits - 1).

    Returns (wq uint32 (V, D * bits / 32), scales uint16 bf16 bits (V, D / G),
    biases uint16 bf16 bits (V, D / G)).  This prepares inputs; the loss
    arithmetic on them lives in the kernels and in the oracle."""
    V, D = W.shape
    if D % group_size or bits not in (2, 4, 8):
        raise ValueError("D must be a multiple of group_size and bits one of 2, 4, 8")
    ng = D // group_size
    wq = np.empty((V, D * bits // 32), dtype=np.uint32)
    sc = np.empty((V, ng), dtype=np.uint16)
    bi = np.empty((V, ng), dtype=np.uint16)
    levels = float(2 ** bits - 1)
    for r0 in range(0, V, CHUNK_ROWS):
        r1 = min(V, r0 + CHUNK_ROWS)
        g = W[r0:r1].astype(np.float32).reshape(r1 - r0, ng, group_size)
        lo = g.min(axis=2)
        hi = g.max(axis=2)
        sc[r0:r1] = round_to_bf16_bits(np.maximum((hi - lo) / levels, 1e-12).astype(np.float32))
        bi[r0:r1] = round_to_bf16_bits(lo)
        scale = bf16_bits_to_f32(sc[r0:r1])[:, :, None]
        bias = bf16_bits_to_f32(bi[r0:r1])[:, :, None]
        q = np.clip(np.rint((g - bias) / scale), 0, levels).astype(np.uint32)
        wq[r0:r1] = pack_codes(q.reshape(r1 - r0, D), bits)
    return wq, sc, bi


def generate_quantized(w: Workload | str, bits: int = 4, group_size: int = 64,
                       N: int | None = None, V: int | None = None, D: int | None = None):
    """(H bf16 bits, (wq, scales, biases), y) for workload `w` with its W (drawn in
    fp32 by the same recipe) quantised by quantize_affine."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    N = w.N if N is None else N
    V = w.V if V is None else V
    D = w.D if D is None else D
    H = _fill_rows(N, D, w.seed, _S_H, "bf16", None)
    Wf = _fill_rows(V, D, w.seed, _S_W, "fp32", row_scales(V, D, w.seed, w.w_scale))
    y = targets(N, V, w.seed, w.targets)
    return H, quantize_affine(Wf, bits, group_size), y
