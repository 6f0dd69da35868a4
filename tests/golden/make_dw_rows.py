"""Writes the oracle's sampled dW rows for the full-size backward checks.

    python tests/golden/make_dw_rows.py [workload ...]

Row j of dW = dZ^T H needs the log-sum-exp of every token (a whole logits row
each), which at N=8192, V=151936, D=4096 takes the fp64 oracle minutes on a
few host cores; so the values are computed once, by this script, and stored
beside it as dw_rows_<workload>.npz.  Only the seeded input generators and
the oracle are used (no value comes from the CUDA path).  Each file records
the SHA-256 of the inputs it was computed from, which the GPU test checks
before comparing.

Gradient: of the mean loss, g_i = float32(1 / N) (the scale the library
applies on the device), as differentiated in section 1 of D. Ineshin, "Een
gefuseerde forward-kernel voor lineaire cross-entropy op Apple-GPU's" (2026):
dZ_ij = g_i (softmax(Z_i)_j - [j == y_i]), dW = dZ^T H.  Stored: dW and its
magnitude bW = |dZ|^T |H| for the selected rows (fp32 is ample for a 2^-8
relative bound), and every token's lse.
"""
import hashlib
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from linear_cross_entropy_bf16_b200 import synth  # noqa: E402

# chunk edges of the library's backward (32768 vocabulary rows per chunk) are
# where a sampled row is most informative; the rest are seeded
CHUNK = 32768


def input_sha256(H, W, y) -> str:
    h = hashlib.sha256()
    for a in (H, W, y):
        h.update(np.ascontiguousarray(a).tobytes())
    return h.hexdigest()


def vocab_rows(V: int, y: np.ndarray, seed: int) -> np.ndarray:
    rows = {0, 1, 2, V - 2, V - 1}
    for e in range(CHUNK, V, CHUNK):
        rows.update((e - 1, e))
    # rows that are some token's target, including the most frequent one
    vals, counts = np.unique(y, return_counts=True)
    rows.add(int(vals[np.argmax(counts)]))
    rows.update(int(v) for v in y[:2])
    rng = np.random.default_rng([seed, 77])
    while len(rows) < 28:
        rows.add(int(rng.integers(0, V)))
    return np.array(sorted(rows), dtype=np.int64)


def make(name: str) -> str:
    w = synth.WORKLOADS[name]
    H, W, y = synth.generate(name)
    rows = vocab_rows(w.V, y, w.seed)
    g = float(np.float32(1.0 / w.N))
    t0 = time.perf_counter()
    out = oracle.grad_weight_rows(H, W, y, g, rows)
    secs = time.perf_counter() - t0
    path = os.path.join(HERE, f"dw_rows_{name}.npz")
    np.savez_compressed(path, workload=name, input_sha256=input_sha256(H, W, y), g=g,
                        vocab_rows=rows, dW=out["dW"].astype(np.float32),
                        bW=out["bW"].astype(np.float32), lse=out["lse"])
    print(f"{name}: {len(rows)} rows in {secs:.0f} s on {oracle.max_threads()} threads -> {path}")
    return path


if __name__ == "__main__":
    names = sys.argv[1:] or ["n8192_v151936_d4096", "n4096_v128256_d4096_zipf"]
    for n in names:
        make(n)
