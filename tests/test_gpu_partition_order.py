"""The partition-aware order of the pair kernel's units, on a B200.

Forwards with at least 16 units per CTA pair run in this order once the
device's L2 partitions have been mapped (by the first such forward).  Only
which pair computes which unit changes, so the results must equal the
oracle's within the usual bounds and be bitwise reproducible, and the
two-stage forward must agree with the one-launch forward bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_bf16_b200 import synth
from tests.flce_testing import compare, run, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_cross_entropy_bf16_b200 import build
    build.build()
    oracle.build()


# 32 (or 32 ragged) token blocks in two raster groups x 37 slabs: 16 units per
# pair on 74 pairs.  The oracle checks a seeded sample of rows (all V and D).
SHAPES = [(8192, 40000, 4096), (8000, 40100, 4096)]


def sample_rows(N, k=192, seed=0):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, N - 1], rng.choice(N, k, replace=False)]))


@pytest.mark.parametrize("N,V,D", SHAPES)
def test_partition_order_sampled_rows(N, V, D):
    import linear_cross_entropy_bf16_b200 as flce
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    p = flce.plan(N, V, D, sm_count=sms)
    assert p["ctas_per_unit"] == 2 and p["token_blocks"] > p["group_blocks"]
    assert p["units"] >= 16 * (p["grid"] // 2)
    H, W, y = synth.random_inputs(N, V, D, seed=N + V + D)
    first = run(H, W, y)    # maps the partitions if no forward has yet
    second = run(H, W, y)
    pairs = flce.partition_map()
    if pairs is not None:
        assert min(pairs) >= 1 and sum(pairs) <= sms // 2
    rows = sample_rows(N)
    ref = oracle.forward(H[rows], W, y[rows])
    compare(second, ref, rows=rows)
    assert abs(second["mean"] - float(np.mean(second["loss"]))) <= 1e-6 * abs(second["mean"])
    for k in ("loss", "lse", "target"):
        assert np.array_equal(first[k], second[k]), k
    assert first["mean"] == second["mean"]


def test_partition_order_two_stage_equals_forward():
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = SHAPES[0]
    H, W, y = synth.random_inputs(N, V, D, seed=77)
    Hd, Wd, yd = to_device(H, W, y)
    one = flce.forward(Hd, Wd, yd)
    ws = torch.empty(flce.workspace_size(N, V, D), dtype=torch.uint8, device="cuda")
    loss, lse, tgt = (torch.empty(N, device="cuda") for _ in range(3))
    mean = torch.empty((), device="cuda")
    flce.partials(Hd, Wd, yd, tgt, ws)
    flce.merge(yd, V, loss, lse, tgt, mean, ws)
    assert flce.check(ws) == flce.OK
    for x, z in zip(one, (loss, lse, tgt, mean)):
        assert torch.equal(x, z)


def test_partition_map_is_taken_on_b200():
    """On B200 the latency probe finds two partitions with pairs on both."""
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = SHAPES[0]
    H, W, y = synth.random_inputs(N, V, D, seed=5)
    run(H, W, y)
    pairs = flce.partition_map()
    assert pairs is not None and pairs[0] >= 1 and pairs[1] >= 1
