"""The forward and the backward captured into CUDA graphs and replayed.

Every call enqueues only stream work (a header reset and kernel launches) and
does no host synchronisation or allocation, so after one eager call (which
sets the kernels' shared-memory limits and caches the device's occupancy) a
call can be captured once and replayed on new contents of the same buffers.
Replays must match eager calls bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_bf16_b200 import synth
from tests.flce_testing import compare, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_cross_entropy_bf16_b200 import build
    build.build()
    oracle.build()


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_forward_graph_replay_matches_eager(dtype):
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 700, 9000, 128
    batches = [synth.random_inputs(N, V, D, seed=s, dtype=dtype) for s in (71, 72, 73)]
    H, W, y = to_device(*batches[0])
    ws = torch.empty(flce.workspace_size(N, V, D, H.dtype), dtype=torch.uint8, device="cuda")
    out = {k: torch.empty(N, device="cuda") for k in ("loss", "lse", "target_logit")}
    out["mean"] = torch.empty((), device="cuda")
    flce.forward(H, W, y, out=out, workspace=ws)          # eager warm-up
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        flce.forward(H, W, y, out=out, workspace=ws)
    for Hn, Wn, yn in batches[1:]:
        Hs, Ws, ys = to_device(Hn, Wn, yn)
        H.copy_(Hs), W.copy_(Ws), y.copy_(ys)
        g.replay()
        torch.cuda.synchronize()
        eager = flce.forward(Hs, Ws, ys, check=True)
        for key, e in zip(("loss", "lse", "target_logit", "mean"), eager):
            assert torch.equal(out[key], e), key
        assert flce.check(ws) == flce.OK
        ref = oracle.forward(Hn, Wn, yn)
        gpu = {"loss": out["loss"].cpu().double().numpy(), "lse": out["lse"].cpu().double().numpy(),
               "target": out["target_logit"].cpu().double().numpy(), "mean": float(out["mean"].item())}
        compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))


def test_backward_graph_replay_matches_eager():
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 400, 20000, 64
    H, W, y = to_device(*synth.random_inputs(N, V, D, seed=74))
    _, lse, _, _ = flce.forward(H, W, y, check=True)
    ws = torch.empty(flce.backward_workspace_size(N, V, D), dtype=torch.uint8, device="cuda")
    out = {"dH": torch.empty(N, D, device="cuda"), "dW": torch.empty(V, D, device="cuda")}
    flce.backward(H, W, y, lse, None, 1.0 / N, out=out, workspace=ws)   # eager warm-up
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        flce.backward(H, W, y, lse, None, 1.0 / N, out=out, workspace=ws)
    H2, W2, y2 = to_device(*synth.random_inputs(N, V, D, seed=75))
    _, lse2, _, _ = flce.forward(H2, W2, y2, check=True)
    H.copy_(H2), W.copy_(W2), y.copy_(y2), lse.copy_(lse2)
    g.replay()
    torch.cuda.synchronize()
    dH, dW = flce.backward(H2, W2, y2, lse2, None, 1.0 / N, check=True)
    assert torch.equal(out["dH"], dH) and torch.equal(out["dW"], dW)
    assert flce.check(ws) == flce.OK
