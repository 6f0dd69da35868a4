"""Oracle for the fused linear cross-entropy forward (fp64, CPU).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The product package
never imports this module, and this module never imports the product package.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over rows).  It
writes out the definition from D. Ineshin, "Een gefuseerde forward-kernel voor
lineaire cross-entropy op Apple-GPU's" (2026), section 1:
Z = H W^T and loss_i = logsumexp(Z_i) - Z_{i, y_i}.  This wrapper only builds
the shared object, marshals numpy arrays and raises on error codes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

BF16 = 0
FP32 = 1
FP64 = 2   # only for the oracle's own finite-difference pins

_ERRORS = {-1: "invalid argument", -2: "target outside [0, V)", -3: "out of memory"}


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (no fast-math: fp64 sums stay in order).

    With ORACLE_LIB_PATH set (only the mutation tests do this: they build a
    copy of oracle.c with one planted mistake), that shared object is used
    instead and nothing is compiled here."""
    if os.environ.get("ORACLE_LIB_PATH"):
        return os.environ["ORACLE_LIB_PATH"]
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared",
                               "-std=c11", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            vp, i64, dp = ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p
            lib.oracle_forward_rows.argtypes = [vp, vp, ctypes.c_int, vp, i64, i64, i64,
                                                vp, i64, dp, dp, dp, dp, ctypes.c_int]
            lib.oracle_forward_rows.restype = ctypes.c_int
            lib.oracle_logits_row.argtypes = [vp, vp, ctypes.c_int, i64, i64, i64, dp]
            lib.oracle_logits_row.restype = ctypes.c_int
            lib.oracle_mean.argtypes = [dp, i64]
            lib.oracle_mean.restype = ctypes.c_double
            lib.oracle_max_threads.argtypes = []
            lib.oracle_max_threads.restype = ctypes.c_int
            lib.oracle_backward.argtypes = [vp, vp, ctypes.c_int, vp, dp, i64, i64, i64,
                                            dp, dp, dp, dp, ctypes.c_int]
            lib.oracle_backward.restype = ctypes.c_int
            lib.oracle_grad_logits_row.argtypes = [vp, vp, ctypes.c_int, vp, ctypes.c_double,
                                                   i64, i64, i64, dp]
            lib.oracle_grad_logits_row.restype = ctypes.c_int
            lib.oracle_grad_hidden_rows.argtypes = [vp, vp, ctypes.c_int, vp, dp, i64, i64, i64,
                                                    vp, i64, dp, dp, ctypes.c_int]
            lib.oracle_grad_hidden_rows.restype = ctypes.c_int
            lib.oracle_grad_weight_rows.argtypes = [vp, vp, ctypes.c_int, vp, dp, i64, i64, i64,
                                                    vp, i64, dp, dp, dp, ctypes.c_int]
            lib.oracle_grad_weight_rows.restype = ctypes.c_int
            lib.oracle_dequantize.argtypes = [vp, vp, vp, ctypes.c_int, i64, i64, i64, dp]
            lib.oracle_dequantize.restype = ctypes.c_int
            lib.oracle_forward_quantized_rows.argtypes = [vp, vp, vp, vp, ctypes.c_int, i64, vp,
                                                          i64, i64, i64, vp, i64, dp, dp, dp, dp,
                                                          ctypes.c_int]
            lib.oracle_forward_quantized_rows.restype = ctypes.c_int
            _lib = lib
    return _lib


def _as_storage(a: np.ndarray):
    """Return (contiguous array, dtype code): uint16 holds bf16 bit patterns."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return a, BF16
    if a.dtype == np.float32:
        return a, FP32
    if a.dtype == np.float64:
        return a, FP64
    raise TypeError(f"oracle takes bf16 bits (uint16), float32 or float64, got {a.dtype}")


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def forward(H: np.ndarray, W: np.ndarray, y: np.ndarray, rows=None, nthreads: int = 0):
    """Per-token loss, lse, target logit and row max for ``rows`` (default: all).

    H is (N, D) and W is (V, D), both uint16 bf16 bit patterns or both float32;
    y is int64 of length N.  Returns a dict of float64 arrays indexed like ``rows``.
    """
    lib = _load()
    H, dt_h = _as_storage(H)
    W, dt_w = _as_storage(W)
    if dt_h != dt_w:
        raise TypeError("H and W must share one storage type")
    if H.ndim != 2 or W.ndim != 2 or H.shape[1] != W.shape[1]:
        raise ValueError("H must be (N, D) and W (V, D)")
    y = np.ascontiguousarray(y, dtype=np.int64)
    N, D = H.shape
    V = W.shape[0]
    if y.shape != (N,):
        raise ValueError("y must have length N")
    if rows is None:
        rows_arr, n = None, N
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows_arr.shape[0]
    out = {k: np.empty(n, dtype=np.float64) for k in ("loss", "lse", "target", "max")}
    rc = lib.oracle_forward_rows(_ptr(H), _ptr(W), dt_h, _ptr(y), N, V, D,
                                 _ptr(rows_arr), n, _ptr(out["loss"]), _ptr(out["lse"]),
                                 _ptr(out["target"]), _ptr(out["max"]), int(nthreads))
    if rc != 0:
        raise OracleError(_ERRORS.get(rc, f"oracle error {rc}"))
    return out


def logits_row(H: np.ndarray, W: np.ndarray, i: int) -> np.ndarray:
    """The full fp64 logits row Z_i (only for small V: it is V doubles)."""
    lib = _load()
    H, dt = _as_storage(H)
    W, _ = _as_storage(W)
    V, D = W.shape
    z = np.empty(V, dtype=np.float64)
    rc = lib.oracle_logits_row(_ptr(H), _ptr(W), dt, int(i), V, D, _ptr(z))
    if rc != 0:
        raise OracleError(_ERRORS.get(rc, f"oracle error {rc}"))
    return z


def mean(loss: np.ndarray) -> float:
    """Mean loss over the given per-token losses (sequential fp64 sum / n)."""
    lib = _load()
    loss = np.ascontiguousarray(loss, dtype=np.float64)
    return float(lib.oracle_mean(_ptr(loss), loss.shape[0]))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def backward(H: np.ndarray, W: np.ndarray, y: np.ndarray, g, bounds: bool = False,
             want_dW: bool = True, nthreads: int = 0):
    """Gradients of sum_i g_i loss_i with respect to H and W (fp64).

    g is a per-token array of upstream gradients or a scalar (1/N gives the
    mean loss).  Returns dict with dH (N, D), dW (V, D) and, with bounds=True,
    bH = |dZ| |W| and bW = |dZ|^T |H| (elementwise magnitudes of the sums).
    """
    lib = _load()
    H, dt = _as_storage(H)
    W, dt_w = _as_storage(W)
    if dt != dt_w:
        raise TypeError("H and W must share one storage type")
    N, D = H.shape
    V = W.shape[0]
    y = np.ascontiguousarray(y, dtype=np.int64)
    gv = np.ascontiguousarray(np.broadcast_to(np.asarray(g, dtype=np.float64), (N,)))
    out = {"dH": np.empty((N, D)), "dW": np.empty((V, D)) if want_dW else None}
    if bounds:
        out["bH"] = np.empty((N, D))
        out["bW"] = np.empty((V, D)) if want_dW else None
    rc = lib.oracle_backward(_ptr(H), _ptr(W), dt, _ptr(y), _ptr(gv), N, V, D,
                             _ptr(out["dH"]), _ptr(out["dW"]), _ptr(out.get("bH")),
                             _ptr(out.get("bW")), int(nthreads))
    if rc != 0:
        raise OracleError(_ERRORS.get(rc, f"oracle error {rc}"))
    return out


def grad_logits_row(H: np.ndarray, W: np.ndarray, y: np.ndarray, g_i: float, i: int) -> np.ndarray:
    """dL/dZ_i. for one row (V values)."""
    lib = _load()
    H, dt = _as_storage(H)
    W, _ = _as_storage(W)
    V, D = W.shape
    y = np.ascontiguousarray(y, dtype=np.int64)
    dz = np.empty(V, dtype=np.float64)
    rc = lib.oracle_grad_logits_row(_ptr(H), _ptr(W), dt, _ptr(y), float(g_i), int(i), V, D, _ptr(dz))
    if rc != 0:
        raise OracleError(_ERRORS.get(rc, f"oracle error {rc}"))
    return dz


def grad_hidden_rows(H: np.ndarray, W: np.ndarray, y: np.ndarray, g, rows, nthreads: int = 0):
    """dH (and its magnitude bound bH) for the selected rows only."""
    lib = _load()
    H, dt = _as_storage(H)
    W, _ = _as_storage(W)
    N, D = H.shape
    V = W.shape[0]
    y = np.ascontiguousarray(y, dtype=np.int64)
    gv = np.ascontiguousarray(np.broadcast_to(np.asarray(g, dtype=np.float64), (N,)))
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    dH = np.empty((rows.shape[0], D))
    bH = np.empty((rows.shape[0], D))
    rc = lib.oracle_grad_hidden_rows(_ptr(H), _ptr(W), dt, _ptr(y), _ptr(gv), N, V, D, _ptr(rows),
                                     rows.shape[0], _ptr(dH), _ptr(bH), int(nthreads))
    if rc != 0:
        raise OracleError(_ERRORS.get(rc, f"oracle error {rc}"))
    return {"dH": dH, "bH": bH}


def grad_weight_rows(H: np.ndarray, W: np.ndarray, y: np.ndarray, g, vocab_rows,
                     nthreads: int = 0):
    """dW (and its magnitude bound bW) for the selected vocabulary rows only, plus every
    token's lse.  Costs one full logits row per token (for lse) and one logits column
    per selected vocabulary row."""
    lib = _load()
    H, dt = _as_storage(H)
    W, dt_w = _as_storage(W)
    if dt != dt_w:
        raise TypeError("H and W must share one storage type")
    N, D = H.shape
    V = W.shape[0]
    y = np.ascontiguousarray(y, dtype=np.int64)
    gv = np.ascontiguousarray(np.broadcast_to(np.asarray(g, dtype=np.float64), (N,)))
    vrows = np.ascontiguousarray(vocab_rows, dtype=np.int64)
    dW = np.empty((vrows.shape[0], D))
    bW = np.empty((vrows.shape[0], D))
    lse = np.empty(N)
    rc = lib.oracle_grad_weight_rows(_ptr(H), _ptr(W), dt, _ptr(y), _ptr(gv), N, V, D, _ptr(vrows),
                                     vrows.shape[0], _ptr(dW), _ptr(bW), _ptr(lse), int(nthreads))
    if rc != 0:
        raise OracleError(_ERRORS.get(rc, f"oracle error {rc}"))
    return {"dW": dW, "bW": bW, "lse": lse}


def _quant_arrays(wq, scales, biases, bits, group_size):
    wq = np.ascontiguousarray(wq)
    scales = np.ascontiguousarray(scales)
    biases = np.ascontiguousarray(biases)
    if wq.dtype != np.uint32 or scales.dtype != np.uint16 or biases.dtype != np.uint16:
        raise TypeError("wq must be uint32 codes, scales and biases uint16 bf16 bit patterns")
    V = wq.shape[0]
    D = wq.shape[1] * (32 // bits)
    if scales.shape != (V, D // group_size) or biases.shape != scales.shape:
        raise ValueError("scales and biases must be (V, D / group_size)")
    return wq, scales, biases, V, D


def dequantize(wq: np.ndarray, scales: np.ndarray, biases: np.ndarray, bits: int = 4,
               group_size: int = 64) -> np.ndarray:
    """The affine-quantised W (V, D) in float64: W_jk = s_jg q_jk + b_jg (g = k // group_size)."""
    lib = _load()
    wq, scales, biases, V, D = _quant_arrays(wq, scales, biases, bits, group_size)
    W = np.empty((V, D), dtype=np.float64)
    rc = lib.oracle_dequantize(_ptr(wq), _ptr(scales), _ptr(biases), int(bits), int(group_size),
                               V, D, _ptr(W))
    if rc != 0:
        raise OracleError(_ERRORS.get(rc, f"oracle error {rc}"))
    return W


def forward_quantized(H: np.ndarray, wq: np.ndarray, scales: np.ndarray, biases: np.ndarray,
                      y: np.ndarray, bits: int = 4, group_size: int = 64, rows=None,
                      nthreads: int = 0):
    """forward() with an affine-quantised head; H is (N, D) bf16 bit patterns (uint16)."""
    lib = _load()
    H = np.ascontiguousarray(H)
    if H.dtype != np.uint16 or H.ndim != 2:
        raise TypeError("H must be (N, D) bf16 bit patterns (uint16)")
    wq, scales, biases, V, D = _quant_arrays(wq, scales, biases, bits, group_size)
    N = H.shape[0]
    if H.shape[1] != D:
        raise ValueError("H and the quantised W disagree on D")
    y = np.ascontiguousarray(y, dtype=np.int64)
    if y.shape != (N,):
        raise ValueError("y must have length N")
    if rows is None:
        rows_arr, n = None, N
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows_arr.shape[0]
    out = {k: np.empty(n, dtype=np.float64) for k in ("loss", "lse", "target", "max")}
    rc = lib.oracle_forward_quantized_rows(_ptr(H), _ptr(wq), _ptr(scales), _ptr(biases), int(bits),
                                           int(group_size), _ptr(y), N, V, D, _ptr(rows_arr), n,
                                           _ptr(out["loss"]), _ptr(out["lse"]), _ptr(out["target"]),
                                           _ptr(out["max"]), int(nthreads))
    if rc != 0:
        raise OracleError(_ERRORS.get(rc, f"oracle error {rc}"))
    return out
