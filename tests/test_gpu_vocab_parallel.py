"""Vocabulary-parallel forward on one GPU: G shards run one after another and
their per-token states are merged, as the ranks of a real run would after
their all-gather.  Checked against the fp64 oracle on every row."""
import math

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


def sharded_forward(Hd, Wd, yd, bounds):
    import linear_cross_entropy_bf16_b200 as flce
    states = [flce.shard_state(Hd, Wd[a:b].contiguous(), yd, a) for a, b in zip(bounds[:-1], bounds[1:])]
    loss, lse, tgt, mean = flce.merge_shards(torch.stack(states).contiguous(), yd, Wd.shape[0], check=True)
    torch.cuda.synchronize()
    return {"loss": loss.cpu().double().numpy(), "lse": lse.cpu().double().numpy(),
            "target": tgt.cpu().double().numpy(), "mean": float(mean.item())}


@pytest.mark.parametrize("N,V,D,bounds", [
    (300, 5000, 128, [0, 2000, 2100, 5000]),          # uneven, one shard of 100 rows
    (129, 70000, 64, [0, 17500, 35000, 52500, 70000]),
    (1000, 1100, 72, [0, 1, 1100]),                    # a one-row shard
])
def test_sharded_matches_oracle(N, V, D, bounds):
    H, W, y = synth.random_inputs(N, V, D, seed=V + len(bounds))
    Hd, Wd, yd = to_device(H, W, y)
    got = sharded_forward(Hd, Wd, yd, bounds)
    ref = oracle.forward(H, W, y)
    compare(got, ref, mean_ref=oracle.mean(ref["loss"]))


def test_one_shard_agrees_with_the_plain_forward():
    import linear_cross_entropy_bf16_b200 as flce
    H, W, y = synth.random_inputs(700, 9000, 256, seed=51)
    Hd, Wd, yd = to_device(H, W, y)
    got = sharded_forward(Hd, Wd, yd, [0, 9000])
    loss, lse, tgt, mean = flce.forward(Hd, Wd, yd)
    assert np.array_equal(got["target"], tgt.cpu().double().numpy())
    assert np.abs(got["lse"] - lse.cpu().double().numpy()).max() <= 1e-5


def test_target_held_by_no_shard_is_flagged():
    import linear_cross_entropy_bf16_b200 as flce
    H, W, y = synth.random_inputs(64, 1000, 64, seed=52)
    y[10] = 1000                       # outside the vocabulary
    Hd, Wd, yd = to_device(H, W, y)
    states = torch.stack([flce.shard_state(Hd, Wd[:600].contiguous(), yd, 0),
                          flce.shard_state(Hd, Wd[600:].contiguous(), yd, 600)]).contiguous()
    with pytest.raises(flce.FlceError) as e:
        flce.merge_shards(states, yd, 1000, check=True)
    assert e.value.status == flce.ERR_TARGET_OUT_OF_RANGE


# ---------------------------------------------------------------- backward
# Each shard's flce_backward_shard gives its rows of dW and its share of dH;
# the shares are summed as the ranks' all-reduce would.  dZ is rounded to
# bf16 (bf16 inputs), so every entry of dH and dW is within 2^-8 of the
# oracle's magnitude bound (bH, bW), as for the single-GPU backward.


@pytest.mark.parametrize("N,V,D,bounds,dtype", [
    (300, 5000, 128, [0, 2000, 2100, 5000], "bf16"),
    (129, 40000, 64, [0, 17500, 35000, 40000], "bf16"),   # shards spanning several chunks
    (200, 3000, 40, [0, 1, 1500, 3000], "fp32"),          # a one-row shard, fp32 inputs
])
def test_sharded_backward_matches_oracle(N, V, D, bounds, dtype):
    import linear_cross_entropy_bf16_b200 as flce
    H, W, y = synth.random_inputs(N, V, D, seed=V + 7 * len(bounds), dtype=dtype)
    Hd, Wd, yd = to_device(H, W, y)
    _, lse, _, _ = flce.forward(Hd, Wd, yd, check=True)
    g = np.random.default_rng(N).uniform(-1, 1, N)
    gd = torch.from_numpy(g.astype(np.float32)).cuda()
    dH = torch.zeros(N, D, dtype=torch.float64, device="cuda")
    dW = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        part, dWs = flce.backward_shard(Hd, Wd[a:b].contiguous(), yd, lse, a, V, gd, check=True)
        dH += part.double()
        dW.append(dWs)
    dW = torch.cat(dW).cpu().double().numpy()
    dH = dH.cpu().numpy()
    ref = oracle.backward(H, W, y, g.astype(np.float32).astype(np.float64), bounds=True)
    for got, r, bnd, name in ((dH, ref["dH"], ref["bH"], "dH"), (dW, ref["dW"], ref["bW"], "dW")):
        err = np.abs(got - r)
        lim = 2.0 ** -8 * bnd + 1e-7
        assert np.all(err <= lim), (name, float((err - lim).max()))
    # dW rows do not depend on how the vocabulary is cut: equal to the unsharded backward's
    _, dW_full = flce.backward(Hd, Wd, yd, lse, gd, check=True)
    assert np.array_equal(dW, dW_full.cpu().double().numpy())


def test_sharded_backward_flags_targets_outside_the_vocabulary():
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 64, 1000, 64
    H, W, y = synth.random_inputs(N, V, D, seed=53)
    Hd, Wd, yd = to_device(H, W, y)
    _, lse, _, _ = flce.forward(Hd, Wd, yd, check=True)
    yb = yd.clone()
    yb[3] = V + 5
    with pytest.raises(flce.FlceError) as e:
        flce.backward_shard(Hd, Wd[600:].contiguous(), yb, lse, 600, V, check=True)
    assert e.value.status == flce.ERR_TARGET_OUT_OF_RANGE


def _vp_backward_rank(rank, world, port, q):
    """One rank of backward_vocab_parallel on CUDA tensors (gloo carries the all-reduce,
    so both ranks can share the one GPU; no kernel of one rank waits on the other)."""
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import linear_cross_entropy_bf16_b200 as flce
        from linear_cross_entropy_bf16_b200 import synth as sy
        from tests.flce_testing import to_device as td
        N, V, D = 256, 20000, 128
        H, W, y = sy.random_inputs(N, V, D, seed=60)
        Hd, Wd, yd = td(H, W, y)
        _, lse, _, _ = flce.forward(Hd, Wd, yd, check=True)
        cut = [0, 12000, V]
        a, b = cut[rank], cut[rank + 1]
        dH, dW = flce.backward_vocab_parallel(Hd, Wd[a:b].contiguous(), yd, lse, a, V,
                                              grad_scale=1.0 / N, check=True)
        torch.cuda.synchronize()
        dH_full, dW_full = flce.backward(Hd, Wd, yd, lse, None, 1.0 / N, check=True)
        q.put((rank, dH.cpu().numpy(), dH_full.cpu().numpy(), bool(torch.equal(dW, dW_full[a:b]))))
    finally:
        dist.destroy_process_group()


def test_backward_vocab_parallel_overlapped_allreduce_two_ranks_one_gpu():
    import socket
    import torch.multiprocessing as mp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_vp_backward_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    # Both sides contract the same bf16 dZ with the same W; only the grouping of
    # the fp32 sums over the vocabulary differs (one sum over all V rows against
    # two shard sums and their all-reduce), so each entry of the two dH differs
    # by at most 2 (V + 1) 2^-24 sum_j |dZ_ij| |W_jk| (the oracle's bH, scaled
    # by 1 + 2^-8 for dZ's rounding to bf16).
    N, V, D = 256, 20000, 128
    H, W, y = synth.random_inputs(N, V, D, seed=60)
    ref = oracle.backward(H, W, y, np.float64(np.float32(1.0 / N)), bounds=True)
    lim = 2 * (V + 1) * 2.0 ** -24 * (1 + 2.0 ** -8) * ref["bH"] + 1e-12
    for rank, dH, dH_full, same_dw in out:
        err = np.abs(dH.astype(np.float64) - dH_full)
        assert np.all(err <= lim), (rank, float((err / lim).max()))
        assert np.linalg.norm(dH - dH_full) / np.linalg.norm(dH_full) < 1e-4
        assert same_dw
