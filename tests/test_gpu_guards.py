"""Every write of the kernels stays inside the buffers it was given, and workspace
contents on entry do not matter.

compute-sanitizer is closed on this machine, so outputs and workspaces are placed
inside larger device buffers whose guard bands (4 KiB before and after) hold a
fixed byte pattern; after each call the bands must be unchanged.  The
workspaces' own bytes are filled with random garbage first (the library
promises that their contents on entry are ignored), and the results are
checked against the oracle.  Shapes are ragged around the tile, row-block and
padding boundaries."""
import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_bf16_b200 import synth
from tests.flce_testing import compare, to_device

pytestmark = pytest.mark.gpu
GUARD = 4096
PATTERN = 0xA5


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_cross_entropy_bf16_b200 import build
    build.build()
    oracle.build()


class Guarded:
    """Device buffers placed between two guard bands of a fixed byte pattern."""

    def __init__(self):
        self.blocks = []

    def tensor(self, shape, dtype, garbage=False):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        raw = torch.full((n + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        inner = raw[GUARD:GUARD + n]
        if garbage:
            inner.copy_(torch.randint(0, 256, (n,), dtype=torch.uint8, device="cuda"))
        self.blocks.append(raw)
        return inner.view(dtype).view(shape) if shape != () else inner.view(dtype).view(())

    def check(self):
        torch.cuda.synchronize()
        for raw in self.blocks:
            head, tail = raw[:GUARD], raw[-GUARD:]
            assert bool((head == PATTERN).all()) and bool((tail == PATTERN).all()), "write outside a buffer"


def outputs(g, N, with_sum=False):
    out = {k: g.tensor((N,), torch.float32) for k in ("loss", "lse", "target_logit")}
    out["mean"] = g.tensor((), torch.float32)
    if with_sum:
        out["sum"] = g.tensor((), torch.float32)
    return out


def as_np(out):
    return {"loss": out["loss"].cpu().double().numpy(), "lse": out["lse"].cpu().double().numpy(),
            "target": out["target_logit"].cpu().double().numpy(), "mean": float(out["mean"].item())}


@pytest.mark.parametrize("dtype,N,V,D", [("bf16", 1, 300, 64), ("bf16", 31, 1000, 128),
                                         ("bf16", 129, 2047, 72), ("bf16", 300, 5000, 256),
                                         ("fp32", 3, 700, 40), ("fp32", 257, 1500, 100)])
def test_forward_writes_stay_in_bounds(dtype, N, V, D):
    import linear_cross_entropy_bf16_b200 as flce
    H, W, y = synth.random_inputs(N, V, D, seed=N + V, dtype=dtype)
    Hd, Wd, yd = to_device(H, W, y)
    g = Guarded()
    ws = g.tensor((flce.workspace_size(N, V, D, Hd.dtype),), torch.uint8, garbage=True)
    out = outputs(g, N, with_sum=True)
    flce.forward_strided(Hd, Wd, yd, out=out, workspace=ws, check=True)
    g.check()
    ref = oracle.forward(H, W, y)
    compare(as_np(out), ref, mean_ref=oracle.mean(ref["loss"]))
    # the same workspace again, now holding the previous call's state
    out2 = outputs(g, N)
    flce.forward(Hd, Wd, yd, out=out2, workspace=ws, check=True)
    g.check()
    assert torch.equal(out2["loss"], out["loss"]) and torch.equal(out2["mean"], out["mean"])


def test_backward_and_shards_write_in_bounds():
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 200, 3000, 64
    H, W, y = synth.random_inputs(N, V, D, seed=5)
    Hd, Wd, yd = to_device(H, W, y)
    g = Guarded()
    out = outputs(g, N)
    flce.forward(Hd, Wd, yd, out=out, check=True)
    bws = g.tensor((flce.backward_workspace_size(N, V, D),), torch.uint8, garbage=True)
    grads = {"dH": g.tensor((N, D), torch.float32), "dW": g.tensor((V, D), torch.float32)}
    flce.backward(Hd, Wd, yd, out["lse"], None, 1.0 / N, out=grads, workspace=bws, check=True)
    g.check()
    ref = oracle.backward(H, W, y, np.float64(np.float32(1.0 / N)), bounds=True)
    for k, b in (("dH", "bH"), ("dW", "bW")):
        err = np.abs(grads[k].cpu().double().numpy() - ref[k])
        assert np.all(err <= 2.0 ** -8 * ref[b] + 1e-7)
    # vocabulary shards: per-shard workspace and state, then the merge
    states = []
    for a, b in ((0, 1100), (1100, V)):
        sws = g.tensor((flce.workspace_size(N, b - a, D),), torch.uint8, garbage=True)
        states.append(flce.shard_state(Hd, Wd[a:b].contiguous(), yd, a, workspace=sws))
    g.check()
    loss, lse, tgt, mean = flce.merge_shards(torch.stack(states).contiguous(), yd, V, check=True)
    assert torch.allclose(loss, out["loss"], atol=1e-5, rtol=0)


@pytest.mark.parametrize("N", [70, 9])
def test_quantized_writes_in_bounds(N):
    import linear_cross_entropy_bf16_b200 as flce
    V, D, bits, G = 17000, 128, 4, 64       # two chunks of the 16384-row expansion
    H, Wf, y = synth.random_inputs(N, V, D, seed=6, dtype="fp32")
    H = synth.round_to_bf16_bits(H)
    wq, sc, bi = synth.quantize_affine(Wf, bits, G)
    dev = torch.device("cuda:0")
    Hd = torch.from_numpy(H).view(torch.bfloat16).to(dev)
    args = (torch.from_numpy(wq.view(np.int32)).to(dev), torch.from_numpy(sc).view(torch.bfloat16).to(dev),
            torch.from_numpy(bi).view(torch.bfloat16).to(dev), torch.from_numpy(y).to(dev))
    g = Guarded()
    ws = g.tensor((flce.quantized_workspace_size(N, V, D, bits, G),), torch.uint8, garbage=True)
    out = outputs(g, N, with_sum=True)
    flce.forward_quantized(Hd, *args, bits, G, out=out, workspace=ws, check=True)
    g.check()
    ref = oracle.forward_quantized(H, wq, sc, bi, y, bits, G)
    compare(as_np(out), ref, mean_ref=oracle.mean(ref["loss"]))
