"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small shapes are compared on every row; they span several 128-token blocks,
several 256-column vocab tiles and slabs, and ragged N, V and D tails.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_bf16_b200 import synth
from tests.flce_testing import LOSS_TOL, compare, check_properties, run, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_cross_entropy_bf16_b200 import build
    build.build()
    oracle.build()


SHAPES = [
    # N, V, D
    (1, 1, 8), (7, 2, 16), (129, 127, 64), (255, 129, 72), (128, 255, 64), (200, 257, 128),
    (300, 1000, 256), (129, 2047, 64), (513, 3000, 8), (64, 4097, 136), (1000, 600, 1024),
    (257, 20000, 64),
]


@pytest.mark.parametrize("N,V,D", SHAPES)
def test_bf16_shapes_every_row(N, V, D):
    H, W, y = synth.random_inputs(N, V, D, seed=N * 7 + V + D)
    gpu = run(H, W, y)
    ref = oracle.forward(H, W, y)
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))


@pytest.mark.parametrize("N,V,D", [(1, 1, 1), (5, 3, 7), (130, 300, 33), (256, 2048, 256), (70, 5000, 100)])
def test_fp32_shapes_every_row(N, V, D):
    H, W, y = synth.random_inputs(N, V, D, seed=N + V + D, dtype="fp32")
    gpu = run(H, W, y)
    ref = oracle.forward(H, W, y)
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))


@pytest.mark.parametrize("where", ["first", "last", "last_ragged_tile", "one_column"])
def test_target_positions(where):
    N, V, D = 300, 1100, 64          # 5 tiles, the last holds 76 columns
    H, W, y = synth.random_inputs(N, V, D, seed=3)
    y = {"first": np.zeros(N), "last": np.full(N, V - 1),
         "last_ragged_tile": np.random.default_rng(0).integers(1024, V, N),
         "one_column": np.full(N, 517)}[where].astype(np.int64)
    gpu = run(H, W, y)
    ref = oracle.forward(H, W, y)
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))


def test_stress_scale_logits():
    """Row scales log-uniform in [0.1, 10]/sqrt(D): logits up to ~+-50 stress the online max."""
    H, W, y = synth.generate("stress_n16384_v262144_d2048", N=384, V=9000, D=256)
    gpu = run(H, W, y)
    ref = oracle.forward(H, W, y)
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))


def test_zero_weights_give_log_V():
    N, V, D = 130, 3000, 64
    H, _, y = synth.random_inputs(N, V, D, seed=5)
    W = np.zeros((V, D), dtype=np.uint16)
    gpu = run(H, W, y)
    assert np.all(gpu["target"] == 0.0)
    np.testing.assert_allclose(gpu["loss"], math.log(V), atol=1e-5)


def test_dominant_target():
    V, D = 700, 64
    rng = np.random.default_rng(1)
    W = synth.round_to_bf16_bits(np.sign(rng.standard_normal((V, D))).astype(np.float32))
    y = rng.integers(0, V, 200)
    H = synth.round_to_bf16_bits(0.5 * synth.bf16_bits_to_f32(W[y]))
    gpu = run(H, W, y)
    ref = oracle.forward(H, W, y)
    compare(gpu, ref)
    assert np.all(gpu["loss"] < 1e-3)


def test_deterministic_bitwise():
    import linear_cross_entropy_bf16_b200 as flce
    H, W, y = synth.random_inputs(700, 40000, 256, seed=11)
    Hd, Wd, yd = to_device(H, W, y)
    a = [t.clone() for t in flce.forward(Hd, Wd, yd)]
    b = flce.forward(Hd, Wd, yd)
    for x, z in zip(a, b):
        assert torch.equal(x, z)


def test_partials_then_merge_equals_forward():
    import linear_cross_entropy_bf16_b200 as flce
    H, W, y = synth.random_inputs(333, 5000, 128, seed=12)
    Hd, Wd, yd = to_device(H, W, y)
    ref = flce.forward(Hd, Wd, yd)
    N = 333
    ws = torch.empty(flce.workspace_size(N, 5000, 128), dtype=torch.uint8, device="cuda")
    loss, lse, tgt = (torch.empty(N, device="cuda") for _ in range(3))
    mean = torch.empty((), device="cuda")
    flce.partials(Hd, Wd, yd, tgt, ws)
    flce.merge(yd, 5000, loss, lse, tgt, mean, ws)
    assert flce.check(ws) == flce.OK
    for x, z in zip(ref, (loss, lse, tgt, mean)):
        assert torch.equal(x, z)


def test_out_of_range_targets_flagged():
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 200, 1000, 64
    H, W, y = synth.random_inputs(N, V, D, seed=13)
    y[[3, 150]] = [-1, V]
    Hd, Wd, yd = to_device(H, W, y)
    ws = torch.empty(flce.workspace_size(N, V, D), dtype=torch.uint8, device="cuda")
    loss, lse, tgt, mean = flce.forward(Hd, Wd, yd, workspace=ws)
    assert flce.check(ws) == flce.ERR_TARGET_OUT_OF_RANGE
    loss = loss.cpu().numpy()
    assert np.isnan(loss[3]) and np.isnan(loss[150]) and math.isnan(mean.item())
    good = np.setdiff1d(np.arange(N), [3, 150])
    yv = y.copy()
    yv[[3, 150]] = 0
    ref = oracle.forward(H, W, yv, rows=good)
    assert np.abs(loss[good] - ref["loss"]).max() <= LOSS_TOL
    # the status clears on the next good call with the same workspace
    y2 = torch.from_numpy(yv).cuda()
    flce.forward(Hd, Wd, y2, workspace=ws)
    assert flce.check(ws) == flce.OK


def test_bounded_wait_times_out_and_context_survives():
    import linear_cross_entropy_bf16_b200 as flce
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    assert flce.selftest_wait_timeout(ws, limit_ns=2_000_000) == flce.OK
    assert flce.check(ws) == flce.ERR_TIMEOUT
    H, W, y = synth.random_inputs(64, 500, 64, seed=14)
    gpu = run(H, W, y)
    compare(gpu, oracle.forward(H, W, y))


def test_host_errors_raise():
    import linear_cross_entropy_bf16_b200 as flce
    H = torch.zeros(4, 60, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(10, 60, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(4, dtype=torch.int64, device="cuda")
    with pytest.raises(flce.FlceError) as e:
        flce.forward(H, W, y)
    assert e.value.status == flce.ERR_UNSUPPORTED
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(flce.FlceError):
        flce.forward(H[:, :56].contiguous(), W[:, :56].contiguous(), y, workspace=ws)


def test_empty_batch_is_a_noop():
    import linear_cross_entropy_bf16_b200 as flce
    H = torch.zeros(0, 64, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(10, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(0, dtype=torch.int64, device="cuda")
    loss, lse, tgt, mean = flce.forward(H, W, y)
    assert loss.numel() == 0 and math.isnan(mean.item())


def test_no_N_by_V_allocation():
    """With outputs and workspace supplied, the call allocates nothing on the device."""
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 2048, 64000, 512
    H, W, y = synth.random_inputs(N, V, D, seed=15)
    Hd, Wd, yd = to_device(H, W, y)
    ws = torch.empty(flce.workspace_size(N, V, D), dtype=torch.uint8, device="cuda")
    out = {k: torch.empty(N, device="cuda") for k in ("loss", "lse", "target_logit")}
    out["mean"] = torch.empty((), device="cuda")
    flce.forward(Hd, Wd, yd, out=out, workspace=ws)
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    flce.forward(Hd, Wd, yd, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert torch.cuda.max_memory_allocated() == base
    assert ws.numel() < 4 * N * V / 30


@pytest.mark.parametrize("dtype,y32", [("bf16", False), ("bf16", True), ("fp32", True)])
def test_strided_rows_and_int32_targets(dtype, y32):
    """flce_forward_ex on row slices of wider buffers (row stride > D) with int32/int64 targets."""
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D, pad = 300, 3000, 128, 72
    H, W, y = synth.random_inputs(N, V, D + pad, seed=61, dtype=dtype)
    Hd, Wd, yd = to_device(H, W, y)
    Hs, Ws = Hd[:, pad:], Wd[:, 8:8 + D]            # strided views: rows of D, stride D + pad
    assert Hs.stride(0) == D + pad and not Hs.is_contiguous()
    yy = yd.to(torch.int32) if y32 else yd
    loss, lse, tgt, mean = flce.forward_strided(Hs, Ws, yy, check=True)
    Hc = np.ascontiguousarray(H[:, pad:])
    Wc = np.ascontiguousarray(W[:, 8:8 + D])
    ref = oracle.forward(Hc, Wc, y)
    gpu = {"loss": loss.cpu().double().numpy(), "lse": lse.cpu().double().numpy(),
           "target": tgt.cpu().double().numpy(), "mean": float(mean.item())}
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))
    # identical to the contiguous call on copies
    ref_gpu = flce.forward(Hs.contiguous(), Ws.contiguous(), yd)
    assert torch.equal(ref_gpu[0], loss)


@pytest.mark.parametrize("dtype,N", [("bf16", 1), ("bf16", 31), ("fp32", 3), ("bf16", 32)])
def test_tiny_batches_strided(dtype, N):
    """Fewer than 32 tokens read H from a copy padded with zero rows (bf16: a copy
    kernel; fp32: the split kernel writes the zero rows); with strided rows too."""
    import linear_cross_entropy_bf16_b200 as flce
    V, D, pad = 5000, 256, 24
    H, W, y = synth.random_inputs(N, V, D + pad, seed=62 + N, dtype=dtype)
    Hd, Wd, yd = to_device(H, W, y)
    Hs = Hd[:, pad:]
    loss, lse, tgt, mean = flce.forward_strided(Hs, Wd[:, :D], yd, check=True)
    ref = oracle.forward(np.ascontiguousarray(H[:, pad:]), np.ascontiguousarray(W[:, :D]), y)
    gpu = {"loss": loss.cpu().double().numpy(), "lse": lse.cpu().double().numpy(),
           "target": tgt.cpu().double().numpy(), "mean": float(mean.item())}
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))


# ---------------------------------------------------------------- fp32 inputs
# fp32 H and W are split into bf16 hi = bf16(x), lo = bf16(x - hi) and
# contracted as hi*hi + hi*lo + lo*hi on the tensor cores.  Per product the
# dropped lo*lo term and the two rounding residues of the lo parts are at most
# about 3 * 2^-16 |h w|; the fp32 accumulation over K = 3 * ceil8(D) terms
# adds at most K * 2^-23 of sum |terms| (a loose bound on any summation
# order).  So |z_gpu - z| <= (3 * 2^-16 + 3 * ceil8(D) * 2^-23) * sum_k |h_k w_k|.


def split_error_bound(H, W, y):
    D = H.shape[1]
    Dp = (D + 7) // 8 * 8
    s = np.abs(H.astype(np.float64) * W[y].astype(np.float64)).sum(axis=1)
    return (3 * 2.0 ** -16 + 3 * Dp * 2.0 ** -23) * s


@pytest.mark.parametrize("N,V,D", [(129, 300, 4096), (513, 3000, 9), (300, 2000, 1000), (2, 70000, 24)])
def test_fp32_more_shapes_every_row(N, V, D):
    """Ragged D (not a multiple of 8), long D, many vocab slabs, a single CTA tile."""
    H, W, y = synth.random_inputs(N, V, D, seed=N * 3 + V + D, dtype="fp32")
    gpu = run(H, W, y)
    ref = oracle.forward(H, W, y)
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))


def test_fp32_target_logit_within_split_bound():
    """The target logit is one contraction; its error must respect the derived bound,
    and stay far below what rounding the fp32 inputs to bf16 would cost."""
    N, V, D = 512, 4000, 256
    H, W, y = synth.random_inputs(N, V, D, seed=77, dtype="fp32")
    gpu = run(H, W, y)
    ref = oracle.forward(H, W, y)
    err = np.abs(gpu["target"] - ref["target"])
    bound = split_error_bound(H, W, y)
    assert np.all(err <= bound), float((err / bound).max())
    # rounding H and W to bf16 first would give target-logit errors of about
    # 2^-9 sqrt(sum (h w)^2) ~ 2e-3 rms here; the split gives about 2^-16 of it
    assert err.max() < 2e-4


def test_fp32_stress_scale_logits():
    """fp32 rows scaled log-uniformly over [0.1, 10]: logits up to ~+-50."""
    N, V, D = 384, 9000, 256
    H, W, y = synth.random_inputs(N, V, D, seed=19, dtype="fp32")
    sig = np.exp(np.random.default_rng(19).uniform(math.log(0.1), math.log(10.0), V)).astype(np.float32)
    W = (W * sig[:, None]).astype(np.float32)
    gpu = run(H, W, y)
    ref = oracle.forward(H, W, y)
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))


def test_fp32_unaligned_strided_rows():
    """fp32 row slices at a 4-byte (not 16-byte) offset with an odd row stride:
    the split kernel's scalar-load path."""
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 260, 1500, 45
    H, W, y = synth.random_inputs(N, V, D + 3, seed=23, dtype="fp32")
    Hd, Wd, yd = to_device(H, W, y)
    Hs, Ws = Hd[:, 1:1 + D], Wd[:, 3:3 + D]
    assert Hs.stride(0) == D + 3 and Hs.data_ptr() % 16 != 0
    loss, lse, tgt, mean = flce.forward_strided(Hs, Ws, yd.to(torch.int32), check=True)
    ref = oracle.forward(np.ascontiguousarray(H[:, 1:1 + D]), np.ascontiguousarray(W[:, 3:3 + D]), y)
    gpu = {"loss": loss.cpu().double().numpy(), "lse": lse.cpu().double().numpy(),
           "target": tgt.cpu().double().numpy(), "mean": float(mean.item())}
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))


# ---------------------------------------------------------------- sum of the losses


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_loss_sum_output(dtype):
    """out_sum of flce_forward_ex, flce_forward_quantized and flce_merge_shards: the
    merge's fp64 total of the per-token losses, rounded once, against the oracle's
    exactly rounded sum (math.fsum of its fp64 losses), within the mean's relative bar."""
    import linear_cross_entropy_bf16_b200 as flce
    from tests.flce_testing import MEAN_RTOL
    N, V, D = 700, 3000, 128
    H, W, y = synth.random_inputs(N, V, D, seed=77, dtype=dtype)
    ref = oracle.forward(H, W, y)
    want = math.fsum(ref["loss"].tolist())
    Hd, Wd, yd = to_device(H, W, y)
    total = torch.full((), float("nan"), device="cuda:0")
    loss, _, _, mean = flce.forward_strided(Hd, Wd, yd, out={"sum": total}, check=True)
    got = float(total.item())
    assert abs(got - want) <= MEAN_RTOL * abs(want), (got, want)
    # the same fp64 total as the mean, rounded once each
    assert abs(got - float(mean.item()) * N) <= 1e-6 * abs(got)
    # vocabulary shards merged: the same sum
    states = torch.stack([flce.shard_state(Hd, Wd[a:b].contiguous(), yd, a)
                          for a, b in ((0, 1000), (1000, V))]).contiguous()
    total2 = torch.full((), float("nan"), device="cuda:0")
    flce.merge_shards(states, yd, V, check=True, out_sum=total2)
    assert abs(float(total2.item()) - want) <= MEAN_RTOL * abs(want)


def test_loss_sum_output_quantized():
    import linear_cross_entropy_bf16_b200 as flce
    from tests.flce_testing import MEAN_RTOL
    N, V, D, bits, G = 300, 2000, 128, 4, 64
    H, Wf, y = synth.random_inputs(N, V, D, seed=78, dtype="fp32")
    H = synth.round_to_bf16_bits(H)
    wq, sc, bi = synth.quantize_affine(Wf, bits, G)
    ref = oracle.forward_quantized(H, wq, sc, bi, y, bits, G)
    want = math.fsum(ref["loss"].tolist())
    dev = torch.device("cuda:0")
    Hd = torch.from_numpy(H).view(torch.bfloat16).to(dev)
    total = torch.full((), float("nan"), device=dev)
    flce.forward_quantized(Hd, torch.from_numpy(wq.view(np.int32)).to(dev),
                           torch.from_numpy(sc).view(torch.bfloat16).to(dev),
                           torch.from_numpy(bi).view(torch.bfloat16).to(dev),
                           torch.from_numpy(y).to(dev), bits, G, out={"sum": total}, check=True)
    assert abs(float(total.item()) - want) <= MEAN_RTOL * abs(want)


# Slab counts P on both sides of every batch edge of the merge (batches of 16
# slab states, loaded two batches ahead in three buffers that take turns: the
# merge leaves its loop after the first, second or third buffer of a round).
# N = 64 runs on the single-CTA kernel, where the planner gives one slab per
# vocabulary tile up to 148 tiles; N = 300 on CTA pairs.  V = 256 tiles - 37
# keeps a ragged last tile.
MERGE_SLAB_COUNTS = [(64, t, t) for t in (1, 15, 16, 17, 32, 33, 48, 49, 64, 65, 97, 148)] + \
                    [(300, 5, 5), (300, 17, 17), (300, 33, 33), (300, 148, 37)]


@pytest.mark.parametrize("N,tiles,P", MERGE_SLAB_COUNTS)
def test_fused_merge_every_slab_count(N, tiles, P):
    import linear_cross_entropy_bf16_b200 as flce
    V, D = 256 * tiles - 37, 64
    # the planned P on 148 SMs (the pair kernel's P follows the pairs that are
    # resident on the device, so it is checked for the single-CTA kernel only)
    assert flce.plan(N, V, D)["slabs"] == P
    if N == 64:
        props = torch.cuda.get_device_properties(0)
        assert flce.plan(N, V, D, sm_count=props.multi_processor_count)["slabs"] == min(P, props.multi_processor_count)
    H, W, y = synth.random_inputs(N, V, D, seed=1000 + N + tiles)
    gpu = run(H, W, y)
    ref = oracle.forward(H, W, y)
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))
    # the two-stage forward (flce_merge_kernel) agrees bit for bit
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
