"""GPU parity of flce_forward_host (inputs and results in host memory, W streamed
to the device in 8192-row chunks through two staging buffers) against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_bf16_b200 import synth
from tests.flce_testing import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_cross_entropy_bf16_b200 import build
    build.build()
    oracle.build()


def host(H, W, y, pin=True):
    def t(a):
        x = torch.from_numpy(np.ascontiguousarray(a))
        x = x.view(torch.bfloat16) if a.dtype == np.uint16 else x
        return x.pin_memory() if pin else x
    return t(H), t(W), t(np.asarray(y, dtype=np.int64))


def as_np(res):
    loss, lse, tgt, mean = res
    return {"loss": loss.double().numpy(), "lse": lse.double().numpy(),
            "target": tgt.double().numpy(), "mean": float(mean.item())}


@pytest.mark.parametrize("N,V,D", [(1, 1, 8), (17, 20000, 64), (129, 8192, 64), (300, 20000, 128), (700, 16385, 64),
                                   (64, 30000, 264)])
def test_host_forward_every_row(N, V, D):
    """One chunk, exactly one chunk, ragged chunks, a one-row last chunk, ragged D."""
    import linear_cross_entropy_bf16_b200 as flce
    H, W, y = synth.random_inputs(N, V, D, seed=N + 3 * V + D)
    cs = torch.cuda.Stream()
    res = flce.forward_host(*host(H, W, y), copy_stream=cs, check=True)
    ref = oracle.forward(H, W, y)
    compare(as_np(res), ref, mean_ref=oracle.mean(ref["loss"]))


def test_host_forward_pageable_and_single_stream():
    """Pageable host memory and no copy stream: slower, same results."""
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 257, 17000, 96
    H, W, y = synth.random_inputs(N, V, D, seed=8)
    a = flce.forward_host(*host(H, W, y, pin=False), check=True)
    b = flce.forward_host(*host(H, W, y), copy_stream=torch.cuda.Stream(), check=True)
    for u, v in zip(a, b):
        assert torch.equal(u, v)
    ref = oracle.forward(H, W, y)
    compare(as_np(a), ref, mean_ref=oracle.mean(ref["loss"]))


def test_host_forward_back_to_back_calls_share_a_workspace():
    """Calls issued back to back on one (stream, workspace): each call's copies wait for
    the previous call's kernels, so the results match the device-input forward."""
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 1000, 40000, 256
    batches = [synth.random_inputs(N, V, D, seed=s) for s in (21, 22, 23)]
    W = batches[0][1]
    cs = torch.cuda.Stream()
    ws = torch.empty(flce.host_workspace_size(N, V, D), dtype=torch.uint8, device="cuda")
    outs, keep = [], []
    for H, _, y in batches:
        inputs = host(H, W, y)
        keep.append(inputs)          # host inputs must outlive the asynchronous copies
        outs.append(flce.forward_host(*inputs, workspace=ws, copy_stream=cs))
    torch.cuda.synchronize()
    assert flce.check(ws) == flce.OK
    Wd = torch.from_numpy(W).view(torch.bfloat16).cuda()
    for (H, _, y), res in zip(batches, outs):
        Hd = torch.from_numpy(H).view(torch.bfloat16).cuda()
        dev = flce.forward(Hd, Wd, torch.from_numpy(y).cuda(), check=True)
        np.testing.assert_allclose(res[0].numpy(), dev[0].cpu().numpy(), rtol=0, atol=2e-6)
        np.testing.assert_allclose(res[1].numpy(), dev[1].cpu().numpy(), rtol=0, atol=2e-6)


def test_host_forward_target_check():
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 200, 9000, 64
    H, W, y = synth.random_inputs(N, V, D, seed=4)
    y = y.copy()
    y[5] = V
    with pytest.raises(flce.FlceError):
        flce.forward_host(*host(H, W, y), check=True)
