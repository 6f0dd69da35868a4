"""flce_forward_noalloc: the forward for callers that cannot allocate device memory.

Such callers (code running inside an allocator or memory-pool callback, or a
runtime that owns the whole device memory budget) cannot hand over a
workspace, so this entry point uses a fixed scratch array built into the
library.  The test calls it through the C ABI (ctypes) twice in a row, with
different inputs, and checks each result against the fp64 oracle on every row
and against flce_forward with a caller-supplied workspace, within the
tolerances of the other GPU tests.  The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_bf16_b200 import synth
from tests.flce_testing import LOSS_TOL, LSE_TOL, MEAN_RTOL, TARGET_TOL, compare, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_cross_entropy_bf16_b200 as flce
    from linear_cross_entropy_bf16_b200 import build
    build.build()
    oracle.build()
    L = flce.load_library()
    fn = L.flce_forward_noalloc
    fn.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 3 + [ctypes.c_int] + [ctypes.c_void_p] * 5
    fn.restype = ctypes.c_int
    return L


def call_noalloc(L, H, W, y, dtype_code):
    N, D = H.shape
    V = W.shape[0]
    out = [torch.full((N,), float("nan"), device="cuda") for _ in range(3)] + \
          [torch.full((), float("nan"), device="cuda")]
    st = L.flce_forward_noalloc(H.data_ptr(), W.data_ptr(), y.data_ptr(), N, V, D, dtype_code,
                                *(t.data_ptr() for t in out), torch.cuda.current_stream().cuda_stream)
    assert st == 0, st
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("dtype,shape", [("bf16", (1000, 40000, 512)), ("fp32", (200, 3000, 64))])
def test_noalloc_matches_forward_twice_in_a_row(lib, dtype, shape):
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = shape
    code = flce.BF16 if dtype == "bf16" else flce.FP32
    for seed in (21, 22):      # two calls in a row, the second on different inputs
        H, W, y = synth.random_inputs(N, V, D, seed=seed, dtype=dtype)
        Hd, Wd, yd = to_device(H, W, y)
        got = call_noalloc(lib, Hd, Wd, yd, code)
        # against the oracle on every row
        want = oracle.forward(H, W, y)
        compare({"loss": got[0].cpu().double().numpy(), "lse": got[1].cpu().double().numpy(),
                 "target": got[2].cpu().double().numpy(), "mean": float(got[3].item())},
                want, mean_ref=oracle.mean(want["loss"]))
        # and against the forward with a caller-supplied workspace
        ref = flce.forward(Hd, Wd, yd, check=True)
        torch.cuda.synchronize()
        for g, r, tol in zip(got[:3], ref[:3], (LOSS_TOL, LSE_TOL, TARGET_TOL)):
            assert torch.isfinite(g).all()
            assert (g - r).abs().max().item() <= tol
        assert abs(got[3].item() - ref[3].item()) <= MEAN_RTOL * abs(ref[3].item())


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    import linear_cross_entropy_bf16_b200 as flce
    # 16384 tokens x 512 slab states x 8 bytes already fills the 64 MiB scratch
    assert flce.workspace_size(16384, 262144, 64) > flce.NOALLOC_SCRATCH_BYTES
    H = torch.zeros(16384, 64, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(262144, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(16384, dtype=torch.int64, device="cuda")
    out = {k: torch.empty(16384, device="cuda") for k in ("loss", "lse", "target_logit")}
    out["mean"] = torch.empty((), device="cuda")
    with pytest.raises(flce.FlceError) as e:
        flce.forward_noalloc(H, W, y, out)
    assert e.value.status == flce.ERR_WORKSPACE_TOO_SMALL
    # the largest problem that fits runs, through the Python binding too
    n_max = 16300
    while flce.workspace_size(n_max + 1, 131072, 64) <= flce.NOALLOC_SCRATCH_BYTES:
        n_max += 1
    assert 16000 < n_max < 16384
    H2, W2, y2 = synth.random_inputs(n_max, 131072, 64, seed=23)
    Hd, Wd, yd = to_device(H2, W2, y2)
    out = {k: torch.empty(n_max, device="cuda") for k in ("loss", "lse", "target_logit")}
    out["mean"] = torch.empty((), device="cuda")
    loss, lse, tgt, mean = flce.forward_noalloc(Hd, Wd, yd, out)
    ref = flce.forward(Hd, Wd, yd)
    assert (loss - ref[0]).abs().max().item() <= LOSS_TOL


def test_noalloc_allocates_nothing(lib):
    import linear_cross_entropy_bf16_b200 as flce
    H, W, y = synth.random_inputs(700, 20000, 256, seed=24)
    Hd, Wd, yd = to_device(H, W, y)
    out = [torch.empty(700, device="cuda") for _ in range(3)] + [torch.empty((), device="cuda")]
    call_noalloc(lib, Hd, Wd, yd, flce.BF16)
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    st = lib.flce_forward_noalloc(Hd.data_ptr(), Wd.data_ptr(), yd.data_ptr(), 700, 20000, 256, flce.BF16,
                                  *(t.data_ptr() for t in out), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == 0 and torch.cuda.max_memory_allocated() == base
