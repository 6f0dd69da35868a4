"""Every pairing of contraction kernel and stage layout, on every row against the oracle.

The forward picks its kernel by N (one CTA per 128-token tile for N <= 128,
CTA pairs above) and its pipeline stage layout by the input type and N:
bf16 stages one K block per stage for N <= 256 (bound by streaming W) and
two consecutive K blocks above; fp32 inputs stage the hi and lo blocks of H
and W together (three products); a quantised head stages H beside W's hi and
lo blocks (two products).  D = 200 is a multiple of neither 64 nor 128, so
the last stage of every layout reads K blocks that lie partly or wholly past
D (zero-filled by TMA).
"""
import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_bf16_b200 import synth
from tests.flce_testing import compare, run

pytestmark = pytest.mark.gpu

V, D = 3001, 200


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_cross_entropy_bf16_b200 import build
    build.build()
    oracle.build()


@pytest.mark.parametrize("dtype,N,kernel", [
    ("bf16", 100, "single CTA, one K block per stage"),
    ("bf16", 256, "CTA pair, one K block per stage"),
    ("bf16", 257, "CTA pair, two K blocks per stage"),
    ("bf16", 300, "CTA pair, two K blocks per stage"),
    ("fp32", 100, "single CTA, hi/lo blocks"),
    ("fp32", 300, "CTA pair, hi/lo blocks"),
])
def test_dense_layouts_every_row(dtype, N, kernel):
    import linear_cross_entropy_bf16_b200 as flce
    p = flce.plan(N, V, D, torch.bfloat16 if dtype == "bf16" else torch.float32)
    assert p["ctas_per_unit"] == (1 if "single" in kernel else 2)
    H, W, y = synth.random_inputs(N, V, D, seed=N + 17, dtype=dtype)
    gpu = run(H, W, y)
    ref = oracle.forward(H, W, y)
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))


@pytest.mark.parametrize("N", [100, 300])
def test_quantised_layout_every_row(N):
    import linear_cross_entropy_bf16_b200 as flce
    bits, G = 4, 64
    Dq = 320                       # a multiple of the group size, not of 128
    H, Wf, y = synth.random_inputs(N, V, Dq, seed=N + 23, dtype="fp32")
    H = synth.round_to_bf16_bits(H)
    wq, sc, bi = synth.quantize_affine(Wf, bits, G)
    dev = torch.device("cuda:0")
    args = (torch.from_numpy(H).view(torch.bfloat16).to(dev), torch.from_numpy(wq.view(np.int32)).to(dev),
            torch.from_numpy(sc).view(torch.bfloat16).to(dev), torch.from_numpy(bi).view(torch.bfloat16).to(dev),
            torch.from_numpy(y).to(dev))
    loss, lse, tgt, mean = flce.forward_quantized(*args, bits, G, check=True)
    ref = oracle.forward_quantized(H, wq, sc, bi, y, bits, G)
    gpu = {"loss": loss.cpu().double().numpy(), "lse": lse.cpu().double().numpy(),
           "target": tgt.cpu().double().numpy(), "mean": float(mean.item())}
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))
