"""Fused linear cross-entropy for NVIDIA B200 (sm_100a).

For hidden states H (N, D), an output projection W (V, D) and targets y (N),
computes loss_i = logsumexp(H_i W^T) - H_i . W_{y_i}, the log-sum-exp, the
target logit and the mean loss without ever forming the (N, V) logits
(D. Ineshin, "Een gefuseerde forward-kernel voor lineaire cross-entropy op
Apple-GPU's", 2026, section 1), and the gradients dH, dW from the saved
log-sum-exp.

Entry points: ``forward`` / ``backward`` (bf16 or fp32), ``forward_strided``
(strided rows, int32 targets), ``forward_quantized`` / ``backward_quantized``
(an affine group-quantised head), ``forward_host`` (inputs and results in
host memory), the vocabulary-parallel ``forward_vocab_parallel`` /
``backward_vocab_parallel`` and their per-shard pieces, ``forward_noalloc``,
and the differentiable loss layers ``linear_cross_entropy`` /
``linear_cross_entropy_quantized``.

This module is a thin ctypes binding over ``libflce.so`` (C ABI in
``include/flce.h``): it checks and marshals torch tensors, allocates outputs
and workspace with torch on the current stream, and calls the library.  All
arithmetic runs in the library's CUDA kernels; there is no fallback.  If the
library is missing, calls raise ``FlceError`` (build it with
``python -m linear_cross_entropy_bf16_b200.build``).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "FlceError", "forward", "backward", "partials", "merge", "workspace_size",
    "shard_state", "merge_shards", "forward_vocab_parallel", "forward_strided",
    "backward_shard", "backward_vocab_parallel",
    "linear_cross_entropy", "linear_cross_entropy_quantized",
    "forward_quantized", "quantized_workspace_size", "backward_quantized",
    "backward_quantized_workspace_size", "forward_host", "host_workspace_size",
    "backward_workspace_size", "plan", "check",
    "status_string", "selftest_wait_timeout", "library_path", "load_library",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libflce.so")
_lock = threading.RLock()
_lib = None

# flce_dtype
BF16 = 0
FP32 = 1
# flce_index_dtype
INDEX_INT64 = 0
INDEX_INT32 = 1
# flce_status
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE_TOO_SMALL, ERR_CUDA, \
    ERR_TARGET_OUT_OF_RANGE, ERR_TIMEOUT = range(7)


_STATUS_NAMES = ("ok", "invalid argument", "unsupported device, shape or alignment",
                 "workspace too small", "CUDA error", "target outside [0, V)",
                 "bounded device wait timed out")


class FlceError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        name = _STATUS_NAMES[status] if 0 <= status < len(_STATUS_NAMES) else "unknown status"
        super().__init__(f"{what}: {name} (status {status})")


class ForwardArgs(ctypes.Structure):
    """Mirror of flce_forward_args."""
    _fields_ = [
        ("H", ctypes.c_void_p), ("ldh", ctypes.c_int64), ("W", ctypes.c_void_p),
        ("ldw", ctypes.c_int64), ("y", ctypes.c_void_p), ("y_dtype", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("N", ctypes.c_int64), ("V", ctypes.c_int64),
        ("D", ctypes.c_int64), ("out_loss", ctypes.c_void_p), ("out_lse", ctypes.c_void_p),
        ("out_target_logit", ctypes.c_void_p), ("out_mean", ctypes.c_void_p),
        ("out_sum", ctypes.c_void_p),
    ]


class Plan(ctypes.Structure):
    """Mirror of flce_plan_t."""
    _fields_ = [
        ("N", ctypes.c_int64), ("V", ctypes.c_int64), ("D", ctypes.c_int64),
        ("dtype", ctypes.c_int32), ("block_rows", ctypes.c_int32),
        ("tile_cols", ctypes.c_int32), ("k_block", ctypes.c_int32),
        ("token_blocks", ctypes.c_int64), ("vocab_tiles", ctypes.c_int64),
        ("slabs", ctypes.c_int32), ("slab_base", ctypes.c_int32),
        ("slab_rem", ctypes.c_int32), ("grid", ctypes.c_int32),
        ("units", ctypes.c_int64), ("makespan_tiles", ctypes.c_int64),
        ("workspace_bytes", ctypes.c_size_t), ("ctas_per_unit", ctypes.c_int32),
        ("group_blocks", ctypes.c_int32),
    ]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libflce.so (once).  Raises FlceError if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise FlceError(ERR_UNSUPPORTED, f"{_LIB_PATH} is missing; build it with "
                            "`python -m linear_cross_entropy_bf16_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        vp, i64, sz, st = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
        lib.flce_workspace_size.argtypes = [i64, i64, i64, ctypes.c_int]
        lib.flce_workspace_size.restype = sz
        lib.flce_plan.argtypes = [i64, i64, i64, ctypes.c_int, ctypes.c_int32, ctypes.POINTER(Plan)]
        lib.flce_plan.restype = st
        i32p = ctypes.POINTER(ctypes.c_int32)
        lib.flce_partition_order.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, i32p]
        lib.flce_partition_order.restype = st
        lib.flce_partition_take.argtypes = [ctypes.c_int32] * 4 + [i32p, i32p]
        lib.flce_partition_take.restype = st
        lib.flce_partition_map.argtypes = [i32p]
        lib.flce_partition_map.restype = st
        lib.flce_forward.argtypes = [vp, vp, vp, i64, i64, i64, ctypes.c_int, vp, vp, vp, vp, vp, sz, vp]
        lib.flce_forward.restype = st
        lib.flce_partials.argtypes = [vp, vp, vp, i64, i64, i64, ctypes.c_int, vp, vp, sz, vp]
        lib.flce_partials.restype = st
        lib.flce_merge.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp, sz, vp]
        lib.flce_merge.restype = st
        lib.flce_check.argtypes = [vp, vp]
        lib.flce_check.restype = st
        lib.flce_status_string.argtypes = [ctypes.c_int]
        lib.flce_status_string.restype = ctypes.c_char_p
        lib.flce_selftest_wait_timeout.argtypes = [vp, sz, ctypes.c_uint64, vp]
        lib.flce_selftest_wait_timeout.restype = st
        lib.flce_backward_workspace_size.argtypes = [i64, i64, i64, ctypes.c_int]
        lib.flce_backward_workspace_size.restype = sz
        lib.flce_backward.argtypes = [vp, vp, vp, vp, vp, ctypes.c_float, i64, i64, i64,
                                      ctypes.c_int, vp, vp, vp, sz, vp]
        lib.flce_backward.restype = st
        lib.flce_partials_shard.argtypes = [vp, vp, vp, i64, i64, i64, i64, ctypes.c_int, vp, vp, sz, vp]
        lib.flce_partials_shard.restype = st
        lib.flce_shard_state.argtypes = [vp, i64, i64, i64, vp, vp, sz, vp, vp]
        lib.flce_shard_state.restype = st
        lib.flce_merge_shards_scratch_size.argtypes = [i64]
        lib.flce_merge_shards_scratch_size.restype = sz
        lib.flce_merge_shards.argtypes = [vp, ctypes.c_int32, vp, i64, i64, vp, vp, vp, vp, vp, vp, sz,
                                          vp]
        lib.flce_merge_shards.restype = st
        lib.flce_forward_ex.argtypes = [ctypes.POINTER(ForwardArgs), vp, sz, vp]
        lib.flce_forward_ex.restype = st
        i32 = ctypes.c_int32
        lib.flce_quantized_workspace_size.argtypes = [i64, i64, i64, i32, i32]
        lib.flce_quantized_workspace_size.restype = sz
        lib.flce_forward_quantized.argtypes = [vp, vp, vp, vp, i32, i32, vp, i64, i64, i64,
                                               vp, vp, vp, vp, vp, vp, sz, vp]
        lib.flce_forward_quantized.restype = st
        lib.flce_backward_shard.argtypes = [vp, vp, vp, vp, vp, ctypes.c_float, i64, i64, i64, i64,
                                            i64, ctypes.c_int, vp, vp, vp, sz, vp, vp]
        lib.flce_backward_shard.restype = st
        lib.flce_backward_quantized_workspace_size.argtypes = [i64, i64, i64, i32, i32]
        lib.flce_backward_quantized_workspace_size.restype = sz
        lib.flce_backward_quantized.argtypes = [vp, vp, vp, vp, i32, i32, vp, vp, vp,
                                                ctypes.c_float, i64, i64, i64, vp, vp, sz, vp]
        lib.flce_backward_quantized.restype = st
        lib.flce_forward_host_workspace_size.argtypes = [i64, i64, i64, ctypes.c_int]
        lib.flce_forward_host_workspace_size.restype = sz
        lib.flce_forward_host.argtypes = [vp, vp, vp, i64, i64, i64, ctypes.c_int, vp, vp, vp, vp,
                                          vp, sz, vp, vp]
        lib.flce_forward_host.restype = st
        _lib = lib
        return lib


def status_string(status: int) -> str:
    try:
        return load_library().flce_status_string(int(status)).decode()
    except FlceError:
        return f"status {status}"


def _raise_on(status: int, what: str):
    if status != OK:
        raise FlceError(status, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"H and W must be bfloat16 or float32, got {t.dtype}")


def workspace_size(N: int, V: int, D: int, dtype=torch.bfloat16) -> int:
    code = dtype if isinstance(dtype, int) else (BF16 if dtype == torch.bfloat16 else FP32)
    n = load_library().flce_workspace_size(int(N), int(V), int(D), code)
    if n == 0:
        raise FlceError(ERR_INVALID_ARG, "workspace_size")
    return int(n)


def plan(N: int, V: int, D: int, dtype=torch.bfloat16, sm_count: int = 148) -> dict:
    """The work decomposition the library uses on a device with ``sm_count`` SMs."""
    code = dtype if isinstance(dtype, int) else (BF16 if dtype == torch.bfloat16 else FP32)
    p = Plan()
    _raise_on(load_library().flce_plan(int(N), int(V), int(D), code, int(sm_count), ctypes.byref(p)),
              "plan")
    return p.as_dict()


_side_streams: dict = {}


def _side_stream(device) -> "torch.cuda.Stream":
    """One extra stream per device for collectives that overlap the kernels."""
    key = torch.device(device).index
    if key not in _side_streams:
        _side_streams[key] = torch.cuda.Stream(device)
    return _side_streams[key]


def _event_ptr(event) -> int | None:
    return int(event.cuda_event) if event is not None else None


def _stream_ptr(stream, device) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return int(s.cuda_stream)


def _check_inputs(H, W, y):
    for name, t in (("H", H), ("W", W), ("y", y)):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if H.dim() != 2 or W.dim() != 2 or H.shape[1] != W.shape[1]:
        raise ValueError(f"H must be (N, D) and W (V, D); got {tuple(H.shape)} and {tuple(W.shape)}")
    if H.dtype != W.dtype:
        raise TypeError("H and W must have the same dtype")
    if y.dtype != torch.int64 or y.dim() != 1 or y.shape[0] != H.shape[0]:
        raise ValueError("y must be int64 of shape (N,)")
    if H.device != W.device or H.device != y.device:
        raise ValueError("H, W and y must be on one device")
    return H.shape[0], W.shape[0], H.shape[1], _dtype_code(H)


def _alloc_outputs(N, device, out):
    if out is None:
        out = {}
    f32 = dict(dtype=torch.float32, device=device)
    loss = out.get("loss") if out.get("loss") is not None else torch.empty(N, **f32)
    lse = out.get("lse") if out.get("lse") is not None else torch.empty(N, **f32)
    tgt = out.get("target_logit") if out.get("target_logit") is not None else torch.empty(N, **f32)
    mean = out.get("mean") if out.get("mean") is not None else torch.full((), float("nan"), **f32)
    for t in (loss, lse, tgt, mean):
        if t.dtype != torch.float32 or t.device != device or not t.is_contiguous():
            raise ValueError("outputs must be contiguous float32 tensors on the input device")
    return loss, lse, tgt, mean


def _sum_output(N, device, out):
    """Device pointer of out["sum"] (a 0-d fp32 tensor that receives the sum of the
    losses), or None; with N == 0 the sum is written here as 0."""
    t = (out or {}).get("sum")
    if t is None:
        return None
    if t.dtype != torch.float32 or t.device != device or t.numel() != 1:
        raise ValueError("out['sum'] must be a one-element float32 tensor on the input device")
    if N == 0:
        t.zero_()
    return t.data_ptr()


def _workspace(N, V, D, code, device, workspace):
    need = load_library().flce_workspace_size(int(N), int(V), int(D), code)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    if workspace.device != device or workspace.numel() * workspace.element_size() < need:
        raise FlceError(ERR_WORKSPACE_TOO_SMALL, "forward")
    return workspace


def forward(H: torch.Tensor, W: torch.Tensor, y: torch.Tensor, *, out: dict | None = None,
            workspace: torch.Tensor | None = None, stream=None, check: bool = False):
    """Per-token loss, lse and target logit, and the mean loss.

    H (N, D) and W (V, D) are contiguous CUDA tensors, both bfloat16 or both
    float32; y is int64 (N,).  Returns (loss, lse, target_logit, mean) as fp32
    CUDA tensors (mean is 0-d).  ``out`` may supply any of the output tensors
    by name and ``workspace`` a uint8 tensor of at least ``workspace_size``
    bytes.  The call is asynchronous on ``stream`` (default: current stream);
    ``check=True`` synchronises and raises on device-side errors.
    """
    N, V, D, code = _check_inputs(H, W, y)
    dev = H.device
    loss, lse, tgt, mean = _alloc_outputs(N, dev, out)
    if N == 0:
        return loss, lse, tgt, mean
    ws = _workspace(N, V, D, code, dev, workspace)
    sp = _stream_ptr(stream, dev)
    lib = load_library()
    st = lib.flce_forward(H.data_ptr(), W.data_ptr(), y.data_ptr(), N, V, D, code,
                          loss.data_ptr(), lse.data_ptr(), tgt.data_ptr(), mean.data_ptr(),
                          ws.data_ptr(), ws.numel() * ws.element_size(), sp)
    _raise_on(st, "flce_forward")
    if check:
        _raise_on(lib.flce_check(ws.data_ptr(), sp), "flce_forward (device)")
    return loss, lse, tgt, mean


def backward_workspace_size(N: int, V: int, D: int, dtype=torch.bfloat16) -> int:
    code = dtype if isinstance(dtype, int) else (BF16 if dtype == torch.bfloat16 else FP32)
    n = load_library().flce_backward_workspace_size(int(N), int(V), int(D), code)
    if n == 0:
        raise FlceError(ERR_INVALID_ARG, "backward_workspace_size")
    return int(n)


def backward(H: torch.Tensor, W: torch.Tensor, y: torch.Tensor, lse: torch.Tensor,
             grad: torch.Tensor | None = None, grad_scale: float = 1.0, *,
             out: dict | None = None, workspace: torch.Tensor | None = None, stream=None,
             check: bool = False):
    """Gradients (dH, dW) of sum_i g_i loss_i, g_i = grad_scale * grad[i] (or grad_scale).

    ``lse`` is the forward's log-sum-exp for the same H and W.  Returns fp32
    tensors dH (N, D) and dW (V, D); ``out`` may supply them as "dH" / "dW".
    Use grad_scale = 1/N with grad = None for the mean loss.
    """
    N, V, D, code = _check_inputs(H, W, y)
    dev = H.device
    out = out or {}
    dH = out.get("dH") if out.get("dH") is not None else torch.empty(N, D, dtype=torch.float32, device=dev)
    dW = out.get("dW") if out.get("dW") is not None else torch.empty(V, D, dtype=torch.float32, device=dev)
    for t, shape in ((dH, (N, D)), (dW, (V, D))):
        if t.dtype != torch.float32 or t.device != dev or not t.is_contiguous() or tuple(t.shape) != shape:
            raise ValueError("dH and dW must be contiguous float32 (N, D) and (V, D) tensors")
    if lse.dtype != torch.float32 or lse.shape != (N,) or not lse.is_contiguous() or lse.device != dev:
        raise ValueError("lse must be a contiguous float32 (N,) tensor on the input device")
    if grad is not None and (grad.dtype != torch.float32 or grad.shape != (N,) or not grad.is_contiguous()
                             or grad.device != dev):
        raise ValueError("grad must be a contiguous float32 (N,) tensor on the input device")
    if N == 0:
        dW.zero_()
        return dH, dW
    lib = load_library()
    need = lib.flce_backward_workspace_size(N, V, D, code)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if workspace.numel() * workspace.element_size() < need:
        raise FlceError(ERR_WORKSPACE_TOO_SMALL, "backward")
    sp = _stream_ptr(stream, dev)
    st = lib.flce_backward(H.data_ptr(), W.data_ptr(), y.data_ptr(), lse.data_ptr(),
                           grad.data_ptr() if grad is not None else None, float(grad_scale),
                           N, V, D, code, dH.data_ptr(), dW.data_ptr(), workspace.data_ptr(),
                           workspace.numel() * workspace.element_size(), sp)
    _raise_on(st, "flce_backward")
    if check:
        _raise_on(lib.flce_check(workspace.data_ptr(), sp), "flce_backward (device)")
    return dH, dW


def forward_strided(H: torch.Tensor, W: torch.Tensor, y: torch.Tensor, *, out: dict | None = None,
                    workspace: torch.Tensor | None = None, stream=None, check: bool = False):
    """flce_forward_ex: like forward(), for H and W whose rows are strided (each row
    contiguous, row stride >= D) and int32 or int64 targets.  ``out["sum"]`` (a 0-d
    fp32 tensor) also receives the sum of the losses, from the same fp64 total as the
    mean."""
    for name, t in (("H", H), ("W", W)):
        if not t.is_cuda or t.dim() != 2 or t.stride(1) != 1 or t.stride(0) < t.shape[1]:
            raise ValueError(f"{name} must be a 2-D CUDA tensor with contiguous rows")
    if y.dtype not in (torch.int64, torch.int32) or y.dim() != 1 or not y.is_contiguous() or not y.is_cuda:
        raise ValueError("y must be a contiguous int64 or int32 CUDA tensor")
    if H.dtype != W.dtype or H.shape[1] != W.shape[1] or y.shape[0] != H.shape[0]:
        raise ValueError("shapes or dtypes of H, W and y do not match")
    N, D = H.shape
    V = W.shape[0]
    code = _dtype_code(H)
    dev = H.device
    loss, lse, tgt, mean = _alloc_outputs(N, dev, out)
    sum_ptr = _sum_output(N, dev, out)
    if N == 0:
        return loss, lse, tgt, mean
    ws = _workspace(N, V, D, code, dev, workspace)
    a = ForwardArgs(H.data_ptr(), H.stride(0), W.data_ptr(), W.stride(0), y.data_ptr(),
                    INDEX_INT32 if y.dtype == torch.int32 else INDEX_INT64, code, N, V, D,
                    loss.data_ptr(), lse.data_ptr(), tgt.data_ptr(), mean.data_ptr(), sum_ptr)
    sp = _stream_ptr(stream, dev)
    lib = load_library()
    _raise_on(lib.flce_forward_ex(ctypes.byref(a), ws.data_ptr(), ws.numel() * ws.element_size(), sp),
              "flce_forward_ex")
    if check:
        _raise_on(lib.flce_check(ws.data_ptr(), sp), "flce_forward_ex (device)")
    return loss, lse, tgt, mean


def shard_state(H: torch.Tensor, W_shard: torch.Tensor, y: torch.Tensor, v_offset: int, *,
                workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """This vocabulary shard's per-token state (N, 4) fp32 {m, s, target logit, owned}.

    W_shard holds rows [v_offset, v_offset + V_shard) of the full W; y holds
    global vocabulary ids.  Steps 1 of the vocabulary-parallel forward
    (flce_partials_shard, then flce_shard_state).
    """
    N, Vs, D, code = _check_inputs(H, W_shard, y)
    dev = H.device
    state = torch.zeros(N, 4, dtype=torch.float32, device=dev)
    if N == 0:
        return state
    ws = _workspace(N, Vs, D, code, dev, workspace)
    wsb = ws.numel() * ws.element_size()
    tgt = torch.zeros(N, dtype=torch.float32, device=dev)
    sp = _stream_ptr(stream, dev)
    lib = load_library()
    _raise_on(lib.flce_partials_shard(H.data_ptr(), W_shard.data_ptr(), y.data_ptr(), N, Vs,
                                      int(v_offset), D, code, tgt.data_ptr(), ws.data_ptr(), wsb, sp),
              "flce_partials_shard")
    _raise_on(lib.flce_shard_state(y.data_ptr(), N, Vs, int(v_offset), tgt.data_ptr(),
                                   ws.data_ptr(), wsb, state.data_ptr(), sp), "flce_shard_state")
    return state


def merge_shards(states: torch.Tensor, y: torch.Tensor, V_total: int, *, stream=None,
                 check: bool = False, out_sum: torch.Tensor | None = None):
    """Merge (G, N, 4) shard states (in shard order) into (loss, lse, target_logit, mean);
    ``out_sum`` (a 0-d fp32 tensor) also receives the sum of the losses."""
    if states.dim() != 3 or states.shape[2] != 4 or states.dtype != torch.float32 or not states.is_contiguous():
        raise ValueError("states must be a contiguous float32 (G, N, 4) tensor")
    G, N = states.shape[0], states.shape[1]
    dev = states.device
    f32 = dict(dtype=torch.float32, device=dev)
    loss, lse, tgt = (torch.empty(N, **f32) for _ in range(3))
    mean = torch.full((), float("nan"), **f32)
    sum_ptr = _sum_output(N, dev, {"sum": out_sum})
    if N == 0:
        return loss, lse, tgt, mean
    lib = load_library()
    scratch = torch.empty(lib.flce_merge_shards_scratch_size(N), dtype=torch.uint8, device=dev)
    sp = _stream_ptr(stream, dev)
    _raise_on(lib.flce_merge_shards(states.data_ptr(), G, y.data_ptr(), N, int(V_total),
                                    loss.data_ptr(), lse.data_ptr(), tgt.data_ptr(), mean.data_ptr(),
                                    sum_ptr, scratch.data_ptr(), scratch.numel(), sp),
              "flce_merge_shards")
    if check:
        _raise_on(lib.flce_check(scratch.data_ptr(), sp), "flce_merge_shards (device)")
    return loss, lse, tgt, mean


def forward_vocab_parallel(H: torch.Tensor, W_shard: torch.Tensor, y: torch.Tensor, v_offset: int,
                           V_total: int, group=None, check: bool = False):
    """Vocabulary-parallel forward: this rank holds W rows [v_offset, v_offset + V_shard).

    Every rank of `group` passes the same H and y.  The only exchange is one
    all-gather of the (N, 4) shard states over torch.distributed (NCCL on
    GPUs); shards must be ordered by rank.  Returns (loss, lse, target_logit,
    mean) for the full vocabulary on every rank.
    """
    import torch.distributed as dist
    state = shard_state(H, W_shard, y, v_offset)
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if world > 1:
        # concatenated along dim 0 (accepted by every backend), then viewed as (G, N, 4)
        flat = torch.empty((world * state.shape[0],) + tuple(state.shape[1:]), dtype=state.dtype,
                           device=state.device)
        dist.all_gather_into_tensor(flat, state, group=group)
        gathered = flat.view((world,) + tuple(state.shape))
    else:
        gathered = state.unsqueeze(0)
    return merge_shards(gathered, y, V_total, check=check)


def backward_shard(H: torch.Tensor, W_shard: torch.Tensor, y: torch.Tensor, lse: torch.Tensor,
                   v_offset: int, V_total: int, grad: torch.Tensor | None = None,
                   grad_scale: float = 1.0, *, out: dict | None = None,
                   workspace: torch.Tensor | None = None, stream=None, dh_ready=None,
                   check: bool = False):
    """flce_backward_shard: (dH_partial, dW_shard) for W rows [v_offset, v_offset + V_shard)
    of a V_total-word vocabulary, with lse over the whole vocabulary.  ``dh_ready``
    (a torch.cuda.Event) is recorded once dH_partial is final, before the last dW GEMMs."""
    N, V, D, code = _check_inputs(H, W_shard, y)
    dev = H.device
    out = out or {}
    dH = out.get("dH") if out.get("dH") is not None else torch.empty(N, D, dtype=torch.float32, device=dev)
    dW = out.get("dW") if out.get("dW") is not None else torch.empty(V, D, dtype=torch.float32, device=dev)
    for t, shape in ((dH, (N, D)), (dW, (V, D))):
        if t.dtype != torch.float32 or t.device != dev or not t.is_contiguous() or tuple(t.shape) != shape:
            raise ValueError("dH and dW must be contiguous float32 (N, D) and (V_shard, D) tensors")
    if lse.dtype != torch.float32 or lse.shape != (N,) or not lse.is_contiguous() or lse.device != dev:
        raise ValueError("lse must be a contiguous float32 (N,) tensor on the input device")
    if grad is not None and (grad.dtype != torch.float32 or grad.shape != (N,) or not grad.is_contiguous()
                             or grad.device != dev):
        raise ValueError("grad must be a contiguous float32 (N,) tensor on the input device")
    if N == 0:
        dH.zero_()
        dW.zero_()
        return dH, dW
    lib = load_library()
    need = lib.flce_backward_workspace_size(N, V, D, code)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if workspace.numel() * workspace.element_size() < need:
        raise FlceError(ERR_WORKSPACE_TOO_SMALL, "backward_shard")
    sp = _stream_ptr(stream, dev)
    _raise_on(lib.flce_backward_shard(H.data_ptr(), W_shard.data_ptr(), y.data_ptr(), lse.data_ptr(),
                                      grad.data_ptr() if grad is not None else None, float(grad_scale),
                                      N, V, int(v_offset), int(V_total), D, code, dH.data_ptr(),
                                      dW.data_ptr(), workspace.data_ptr(),
                                      workspace.numel() * workspace.element_size(), sp,
                                      _event_ptr(dh_ready)),
              "flce_backward_shard")
    if check:
        _raise_on(lib.flce_check(workspace.data_ptr(), sp), "flce_backward_shard (device)")
    return dH, dW


def backward_vocab_parallel(H: torch.Tensor, W_shard: torch.Tensor, y: torch.Tensor, lse: torch.Tensor,
                            v_offset: int, V_total: int, grad: torch.Tensor | None = None,
                            grad_scale: float = 1.0, group=None, check: bool = False):
    """Vocabulary-parallel backward: every rank of `group` passes the same H, y and the
    whole-vocabulary lse (from forward_vocab_parallel) and its own W shard.  Returns
    (dH, dW_shard): dH summed over the shards with one all-reduce over
    torch.distributed (NCCL on GPUs), dW_shard this rank's rows of dW."""
    import torch.distributed as dist
    multi = dist.is_initialized() and dist.get_world_size(group) > 1
    if not (multi and H.is_cuda):
        dH, dW = backward_shard(H, W_shard, y, lse, v_offset, V_total, grad, grad_scale, check=check)
        if multi:
            dist.all_reduce(dH, op=dist.ReduceOp.SUM, group=group)
        return dH, dW
    # The all-reduce of dH runs on a side stream as soon as dH is final, while
    # the last dW GEMMs finish on the compute stream.
    main = torch.cuda.current_stream(H.device)
    side = _side_stream(H.device)
    ready = torch.cuda.Event()
    ws = torch.empty(backward_workspace_size(H.shape[0], W_shard.shape[0], H.shape[1], H.dtype),
                     dtype=torch.uint8, device=H.device)
    dH, dW = backward_shard(H, W_shard, y, lse, v_offset, V_total, grad, grad_scale, workspace=ws,
                            stream=main, dh_ready=ready)
    side.wait_event(ready)
    with torch.cuda.stream(side):
        dist.all_reduce(dH, op=dist.ReduceOp.SUM, group=group)
    dH.record_stream(side)
    main.wait_stream(side)
    if check:
        _raise_on(load_library().flce_check(ws.data_ptr(), _stream_ptr(main, H.device)),
                  "backward_vocab_parallel (device)")
    return dH, dW


def partials(H, W, y, target_logit, workspace, stream=None):
    """First stage only (contraction + online (m, s) per vocab slab); see flce_partials."""
    N, V, D, code = _check_inputs(H, W, y)
    if N == 0:
        return
    sp = _stream_ptr(stream, H.device)
    _raise_on(load_library().flce_partials(H.data_ptr(), W.data_ptr(), y.data_ptr(), N, V, D, code,
                                           target_logit.data_ptr(), workspace.data_ptr(),
                                           workspace.numel() * workspace.element_size(), sp),
              "flce_partials")


def merge(y, V, loss, lse, target_logit, mean, workspace, stream=None):
    """Second stage only (combine slab states, loss, mean); see flce_merge."""
    N = y.shape[0]
    if N == 0:
        return
    sp = _stream_ptr(stream, y.device)
    _raise_on(load_library().flce_merge(y.data_ptr(), N, int(V), loss.data_ptr(), lse.data_ptr(),
                                        target_logit.data_ptr(),
                                        mean.data_ptr() if mean is not None else None,
                                        workspace.data_ptr(),
                                        workspace.numel() * workspace.element_size(), sp),
              "flce_merge")


def partition_map(device=None):
    """CTA pairs on the two L2 partitions of the device, as mapped by the first
    forward large enough for the partition-aware order, or None (see
    flce_partition_map)."""
    lib = load_library()
    out = (ctypes.c_int32 * 2)()
    if device is None:
        st = lib.flce_partition_map(out)
    else:
        with torch.cuda.device(device):
            st = lib.flce_partition_map(out)
    return (out[0], out[1]) if st == OK else None


def check(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise ``stream`` and return the status of the last call on ``workspace``."""
    return int(load_library().flce_check(workspace.data_ptr(), _stream_ptr(stream, workspace.device)))


def selftest_wait_timeout(workspace: torch.Tensor, limit_ns: int = 1_000_000, stream=None) -> int:
    """Run the bounded-wait self-test kernel; returns the launch status (read the result with check)."""
    return int(load_library().flce_selftest_wait_timeout(
        workspace.data_ptr(), workspace.numel() * workspace.element_size(), int(limit_ns),
        _stream_ptr(stream, workspace.device)))


# Built-in scratch size of flce_forward_noalloc (FLCE_NOALLOC_SCRATCH_BYTES in include/flce.h).
NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


def forward_noalloc(H: torch.Tensor, W: torch.Tensor, y: torch.Tensor, out: dict, stream=None):
    """flce_forward_noalloc: the forward with the library's built-in scratch.

    For callers that cannot allocate device memory at call time (allocator
    callbacks, runtimes that own the device memory budget): no workspace is
    passed, and the library allocates nothing.  ``out`` must supply all four
    output tensors ("loss", "lse", "target_logit", "mean").  The scratch is
    shared by every call on the device, so calls must be ordered on one stream.
    Raises FlceError(ERR_WORKSPACE_TOO_SMALL) for problems beyond the scratch.
    """
    N, V, D, code = _check_inputs(H, W, y)
    tensors = [out[k] for k in ("loss", "lse", "target_logit", "mean")]
    for t in tensors:
        if t.dtype != torch.float32 or t.device != H.device or not t.is_contiguous():
            raise ValueError("outputs must be contiguous float32 tensors on the input device")
    lib = load_library()
    fn = lib.flce_forward_noalloc
    fn.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 3 + [ctypes.c_int] + [ctypes.c_void_p] * 5
    fn.restype = ctypes.c_int
    st = fn(H.data_ptr(), W.data_ptr(), y.data_ptr(), N, V, D, code,
            *(t.data_ptr() for t in tensors), _stream_ptr(stream, H.device))
    _raise_on(st, "flce_forward_noalloc")
    return tuple(tensors)


def quantized_workspace_size(N: int, V: int, D: int, bits: int = 4, group_size: int = 64) -> int:
    n = load_library().flce_quantized_workspace_size(int(N), int(V), int(D), int(bits), int(group_size))
    if n == 0:
        raise FlceError(ERR_INVALID_ARG, "quantized_workspace_size")
    return int(n)


def forward_quantized(H: torch.Tensor, wq: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor,
                      y: torch.Tensor, bits: int = 4, group_size: int = 64, *, out: dict | None = None,
                      workspace: torch.Tensor | None = None, stream=None, check: bool = False):
    """flce_forward_quantized: the forward with an affine group-quantised head
    W = scales * q + biases (MLX layout: wq (V, D * bits / 32) int32/uint32 codes,
    scales and biases (V, D / group_size) bf16).  Returns (loss, lse, target_logit, mean);
    ``out["sum"]`` (a 0-d fp32 tensor) also receives the sum of the losses."""
    if H.dtype != torch.bfloat16 or H.dim() != 2 or not H.is_contiguous() or not H.is_cuda:
        raise ValueError("H must be a contiguous 2-D bf16 CUDA tensor")
    dev = H.device
    N, D = H.shape
    if wq.dtype not in (torch.int32, torch.uint32) or wq.dim() != 2 or not wq.is_contiguous():
        raise ValueError("wq must be a contiguous 2-D int32/uint32 tensor of packed codes")
    V = wq.shape[0]
    if wq.shape[1] * 32 != D * bits:
        raise ValueError("wq must have D * bits / 32 words per row")
    for name, t in (("scales", scales), ("biases", biases)):
        if (t.dtype != torch.bfloat16 or not t.is_contiguous() or t.device != dev
                or tuple(t.shape) != (V, D // group_size)):
            raise ValueError(f"{name} must be a contiguous bf16 (V, D / group_size) tensor")
    if wq.device != dev or y.device != dev or y.dtype != torch.int64 or y.shape != (N,) \
            or not y.is_contiguous():
        raise ValueError("wq and y must be on H's device; y contiguous int64 of length N")
    loss, lse, tgt, mean = _alloc_outputs(N, dev, out)
    sum_ptr = _sum_output(N, dev, out)
    if N == 0:
        return loss, lse, tgt, mean
    lib = load_library()
    need = quantized_workspace_size(N, V, D, bits, group_size)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    nbytes = workspace.numel() * workspace.element_size()
    sp = _stream_ptr(stream, dev)
    _raise_on(lib.flce_forward_quantized(H.data_ptr(), wq.data_ptr(), scales.data_ptr(),
                                         biases.data_ptr(), int(bits), int(group_size), y.data_ptr(),
                                         N, V, D, loss.data_ptr(), lse.data_ptr(), tgt.data_ptr(),
                                         mean.data_ptr(), sum_ptr, workspace.data_ptr(), nbytes, sp),
              "flce_forward_quantized")
    if check:
        _raise_on(lib.flce_check(workspace.data_ptr(), sp), "flce_forward_quantized (device)")
    return loss, lse, tgt, mean



def backward_quantized_workspace_size(N: int, V: int, D: int, bits: int = 4, group_size: int = 64) -> int:
    n = load_library().flce_backward_quantized_workspace_size(int(N), int(V), int(D), int(bits),
                                                              int(group_size))
    if n == 0:
        raise FlceError(ERR_INVALID_ARG, "backward_quantized_workspace_size")
    return int(n)


def backward_quantized(H: torch.Tensor, wq: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor,
                       y: torch.Tensor, lse: torch.Tensor, grad: torch.Tensor | None = None,
                       grad_scale: float = 1.0, bits: int = 4, group_size: int = 64, *,
                       out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                       stream=None, check: bool = False) -> torch.Tensor:
    """flce_backward_quantized: dH (N, D) fp32 of sum_i g_i loss_i for a frozen
    quantised head (arguments as forward_quantized and backward)."""
    if H.dtype != torch.bfloat16 or H.dim() != 2 or not H.is_contiguous() or not H.is_cuda:
        raise ValueError("H must be a contiguous 2-D bf16 CUDA tensor")
    dev = H.device
    N, D = H.shape
    V = wq.shape[0]
    if wq.dtype not in (torch.int32, torch.uint32) or wq.dim() != 2 or not wq.is_contiguous() \
            or wq.shape[1] * 32 != D * bits:
        raise ValueError("wq must be contiguous (V, D * bits / 32) int32/uint32 codes")
    for name, t in (("scales", scales), ("biases", biases)):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or tuple(t.shape) != (V, D // group_size):
            raise ValueError(f"{name} must be a contiguous bf16 (V, D / group_size) tensor")
    if lse.dtype != torch.float32 or lse.shape != (N,) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 (N,) tensor")
    if grad is not None and (grad.dtype != torch.float32 or grad.shape != (N,) or not grad.is_contiguous()):
        raise ValueError("grad must be a contiguous float32 (N,) tensor")
    if y.dtype != torch.int64 or y.shape != (N,) or not y.is_contiguous():
        raise ValueError("y must be contiguous int64 of length N")
    for t in (wq, scales, biases, y, lse):
        if t.device != dev:
            raise ValueError("all tensors must be on H's device")
    dH = out if out is not None else torch.empty(N, D, dtype=torch.float32, device=dev)
    if dH.dtype != torch.float32 or tuple(dH.shape) != (N, D) or not dH.is_contiguous() or dH.device != dev:
        raise ValueError("out must be a contiguous float32 (N, D) tensor on H's device")
    if N == 0:
        return dH
    lib = load_library()
    need = backward_quantized_workspace_size(N, V, D, bits, group_size)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    sp = _stream_ptr(stream, dev)
    _raise_on(lib.flce_backward_quantized(H.data_ptr(), wq.data_ptr(), scales.data_ptr(),
                                          biases.data_ptr(), int(bits), int(group_size), y.data_ptr(),
                                          lse.data_ptr(), grad.data_ptr() if grad is not None else None,
                                          float(grad_scale), N, V, D, dH.data_ptr(), workspace.data_ptr(),
                                          workspace.numel() * workspace.element_size(), sp),
              "flce_backward_quantized")
    if check:
        _raise_on(lib.flce_check(workspace.data_ptr(), sp), "flce_backward_quantized (device)")
    return dH

def host_workspace_size(N: int, V: int, D: int) -> int:
    n = load_library().flce_forward_host_workspace_size(int(N), int(V), int(D), BF16)
    if n == 0:
        raise FlceError(ERR_INVALID_ARG, "host_workspace_size")
    return int(n)


def forward_host(H: torch.Tensor, W: torch.Tensor, y: torch.Tensor, *, device=None,
                 out: dict | None = None, workspace: torch.Tensor | None = None, stream=None,
                 copy_stream=None, check: bool = False):
    """flce_forward_host: the forward on CPU tensors H (N, D) bf16, W (V, D) bf16 and
    y (N) int64 (pin them for overlap), streaming W to `device` chunk by chunk.

    Returns CPU tensors (loss, lse, target_logit, mean); ``out`` may supply them
    (pinned).  They are valid after `stream` is synchronised (done here when
    ``check`` is set); until then H, W and y must stay alive and unchanged."""
    for name, t in (("H", H), ("W", W), ("y", y)):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CPU tensor")
    if H.dtype != torch.bfloat16 or W.dtype != torch.bfloat16 or H.dim() != 2 or W.dim() != 2 \
            or H.shape[1] != W.shape[1]:
        raise ValueError("H (N, D) and W (V, D) must be bf16 with one D")
    if y.dtype != torch.int64 or y.shape != (H.shape[0],):
        raise ValueError("y must be int64 of shape (N,)")
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    N, D = H.shape
    V = W.shape[0]
    out = out or {}
    pin = torch.cuda.is_available()
    def host(key, shape):
        t = out.get(key)
        return t if t is not None else torch.empty(shape, dtype=torch.float32, pin_memory=pin)
    loss, lse, tgt, mean = host("loss", (N,)), host("lse", (N,)), host("target_logit", (N,)), host("mean", ())
    if N == 0:
        return loss, lse, tgt, mean
    lib = load_library()
    need = host_workspace_size(N, V, D)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    sp = _stream_ptr(stream, dev)
    cp = int(copy_stream.cuda_stream) if copy_stream is not None else None
    _raise_on(lib.flce_forward_host(H.data_ptr(), W.data_ptr(), y.data_ptr(), N, V, D, BF16,
                                    loss.data_ptr(), lse.data_ptr(), tgt.data_ptr(), mean.data_ptr(),
                                    workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                    sp, cp), "flce_forward_host")
    if check:
        _raise_on(lib.flce_check(workspace.data_ptr(), sp), "flce_forward_host (device)")
    return loss, lse, tgt, mean


# ---------------------------------------------------------------- autograd


class _LinearCrossEntropy(torch.autograd.Function):
    """loss = cross_entropy(H W^T, y) with the fused kernels in both directions."""

    @staticmethod
    def forward(ctx, H, W, y, reduction):
        total = torch.empty((), dtype=torch.float32, device=H.device)
        loss, lse, _, mean = forward_strided(H, W, y, out={"sum": total})
        ctx.save_for_backward(H, W, y, lse)
        ctx.reduction = reduction
        if reduction == "mean":
            return mean
        if reduction == "sum":
            return total
        return loss

    @staticmethod
    def backward(ctx, grad_out):
        H, W, y, lse = ctx.saved_tensors
        N = H.shape[0]
        need_h, need_w = ctx.needs_input_grad[0], ctx.needs_input_grad[1]
        if not (need_h or need_w):
            return None, None, None, None
        grad_out = grad_out.float()
        if ctx.reduction == "none":
            g, scale = grad_out.contiguous(), 1.0
        else:
            # the upstream scalar times 1/N (mean) or 1 (sum), applied on the device
            g = grad_out.reshape(1).expand(N).contiguous()
            scale = 1.0 / N if (ctx.reduction == "mean" and N) else 1.0
        dH, dW = backward(H, W, y, lse, g, scale)
        return (dH.to(H.dtype) if need_h else None, dW.to(W.dtype) if need_w else None, None, None)


def linear_cross_entropy(H: torch.Tensor, W: torch.Tensor, y: torch.Tensor,
                         reduction: str = "mean") -> torch.Tensor:
    """Differentiable fused linear cross-entropy: cross_entropy(H @ W.T, y) without the
    (N, V) logits, in the forward (flce_forward) and the backward (flce_backward).

    H (N, D) and W (V, D) bf16 or fp32 on one CUDA device, y (N) int64.  reduction:
    "mean" (default), "sum" or "none" (per-token losses).  Gradients come back in the
    inputs' dtypes (computed in fp32)."""
    if reduction not in ("mean", "sum", "none"):
        raise ValueError("reduction must be 'mean', 'sum' or 'none'")
    if y.dtype == torch.int32:
        y = y.long()
    # the kernels take contiguous rows; a strided view is copied first (the copy
    # is an ordinary differentiable op, so gradients still reach the original)
    return _LinearCrossEntropy.apply(H.contiguous(), W.contiguous(), y.contiguous(), reduction)


class _LinearCrossEntropyQuantized(torch.autograd.Function):
    """The same with a frozen affine-quantised head: gradients for H only."""

    @staticmethod
    def forward(ctx, H, wq, scales, biases, y, bits, group_size, reduction):
        total = torch.empty((), dtype=torch.float32, device=H.device)
        loss, lse, _, mean = forward_quantized(H, wq, scales, biases, y, bits, group_size,
                                               out={"sum": total})
        ctx.save_for_backward(H, wq, scales, biases, y, lse)
        ctx.args = (bits, group_size, reduction)
        if reduction == "mean":
            return mean
        if reduction == "sum":
            return total
        return loss

    @staticmethod
    def backward(ctx, grad_out):
        H, wq, scales, biases, y, lse = ctx.saved_tensors
        bits, group_size, reduction = ctx.args
        none = (None,) * 7
        if not ctx.needs_input_grad[0]:
            return (None,) + none
        N = H.shape[0]
        grad_out = grad_out.float()
        if reduction == "none":
            g, scale = grad_out.contiguous(), 1.0
        else:
            g = grad_out.reshape(1).expand(N).contiguous()
            scale = 1.0 / N if (reduction == "mean" and N) else 1.0
        dH = backward_quantized(H, wq, scales, biases, y, lse, g, scale, bits, group_size)
        return (dH.to(H.dtype),) + none


def linear_cross_entropy_quantized(H: torch.Tensor, wq: torch.Tensor, scales: torch.Tensor,
                                   biases: torch.Tensor, y: torch.Tensor, bits: int = 4,
                                   group_size: int = 64, reduction: str = "mean") -> torch.Tensor:
    """Differentiable loss with a frozen quantised head (MLX affine layout, as
    forward_quantized); only H receives a gradient."""
    if reduction not in ("mean", "sum", "none"):
        raise ValueError("reduction must be 'mean', 'sum' or 'none'")
    if y.dtype == torch.int32:
        y = y.long()
    return _LinearCrossEntropyQuantized.apply(H.contiguous(), wq, scales, biases, y.contiguous(), bits,
                                              group_size, reduction)
