"""The multi-rank (N > 1) benchmark path on CPU: two gloo ranks.

Each rank runs its own batch of tokens against the same W (data-parallel,
weak scaling, no collective on the data path); timings are combined as the
maximum over ranks.  Nothing here touches a GPU.
"""
import hashlib
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from linear_cross_entropy_bf16_b200 import synth
        w = synth.Workload("t", 300, 1000, 64, "bf16", "uniform", "inv_sqrt_d", 9)
        H, W, y = bench.rank_inputs(w, rank)
        digests = [hashlib.sha256(a.tobytes()).hexdigest() for a in (H, W, y)]
        gathered = [None] * world
        dist.all_gather_object(gathered, digests)
        mx = bench.max_over_ranks([rank + 1.0, 10.0 * (world - rank), -1.0], world)
        dist.barrier()
        q.put((rank, gathered, mx))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_W_and_reduce_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    for rank, gathered, mx in out:
        (h0, w0, y0), (h1, w1, y1) = gathered
        assert w0 == w1                 # the projection is replicated
        assert h0 != h1 and y0 != y1    # each rank has its own tokens and targets
        assert mx == [2.0, 20.0, -1.0]  # element-wise max over ranks


def test_weak_scaling_value_counts_all_ranks():
    import bench
    assert bench.weak_scaling_tokens_per_s(1, 8192, 8.0) == pytest.approx(1.024e6)
    assert bench.weak_scaling_tokens_per_s(8, 8192, 8.0) == pytest.approx(8.192e6)
    assert bench.max_over_ranks([1.5, 2.5], 1) == [1.5, 2.5]


def test_reference_arm_under_torchrun_prints_one_line():
    """`--impl reference` under torchrun: rank 0 prints one JSON line, the other rank exits 0."""
    env = dict(os.environ, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={free_port()}", "bench.py", "--gpus", "2",
           "--impl", "reference", "--workload", "tiny_n256_v2048_d256_fp32", "--steps", "2",
           "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    import json
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["e2e"]["h2d_bytes_per_step"] == 0


def _vp_worker(rank, world, port, q):
    """forward_vocab_parallel's exchange on two gloo ranks; the kernel steps are
    replaced by an fp64 restatement so that only the orchestration is under test."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import linear_cross_entropy_bf16_b200 as flce
        rng = np.random.default_rng(7)
        N, V, D = 6, 10, 4
        H = torch.from_numpy(rng.standard_normal((N, D)))
        W = torch.from_numpy(rng.standard_normal((V, D)))
        y = torch.from_numpy(rng.integers(0, V, N))
        cut = [0, 4, 10]
        a, b = cut[rank], cut[rank + 1]

        def fake_state(H_, W_shard, y_, v_offset, **kw):
            z = (H_ @ W_shard.T)
            m = z.max(dim=1).values
            s = torch.exp(z - m[:, None]).sum(dim=1)
            rel = y_ - v_offset
            own = (rel >= 0) & (rel < W_shard.shape[0])
            t = torch.where(own, z[torch.arange(z.shape[0]), rel.clamp(0, W_shard.shape[0] - 1)], 0.0)
            return torch.stack([m, s, t, own.double()], dim=1)

        def fake_merge(states, y_, V_total, **kw):
            m = states[..., 0].max(dim=0).values
            s = (states[..., 1] * torch.exp(states[..., 0] - m)).sum(dim=0)
            lse = m + torch.log(s)
            t = (states[..., 2] * states[..., 3]).sum(dim=0)
            return lse - t, lse, t, (lse - t).mean()

        flce.shard_state = fake_state
        flce.merge_shards = fake_merge
        loss, lse, t, mean = flce.forward_vocab_parallel(H, W[a:b].contiguous(), y, a, V)
        ref = torch.nn.functional.cross_entropy(H @ W.T, y, reduction="none")
        q.put((rank, float((loss - ref).abs().max()), float(mean - ref.mean())))
    finally:
        dist.destroy_process_group()


def test_vocab_parallel_exchange_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_vp_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    for rank, dloss, dmean in out:
        assert dloss < 1e-12 and abs(dmean) < 1e-12


def _vpb_worker(rank, world, port, q):
    """backward_vocab_parallel's all-reduce on two gloo ranks; the kernel step is
    replaced by an fp64 restatement of one shard's dH share and dW rows."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import linear_cross_entropy_bf16_b200 as flce
        rng = np.random.default_rng(8)
        N, V, D = 6, 10, 4
        H = torch.from_numpy(rng.standard_normal((N, D)))
        W = torch.from_numpy(rng.standard_normal((V, D)))
        y = torch.from_numpy(rng.integers(0, V, N))
        lse = torch.logsumexp(H @ W.T, dim=1)
        cut = [0, 3, 10]
        a, b = cut[rank], cut[rank + 1]

        def fake_shard(H_, W_shard, y_, lse_, v_offset, V_total, grad=None, grad_scale=1.0, **kw):
            z = H_ @ W_shard.T
            p = torch.exp(z - lse_[:, None])
            rel = y_ - v_offset
            own = (rel >= 0) & (rel < W_shard.shape[0])
            onehot = torch.zeros_like(p)
            onehot[own, rel[own]] = 1.0
            dz = grad_scale * (p - onehot)
            return dz @ W_shard, dz.T @ H_

        flce.backward_shard = fake_shard
        dH, dW = flce.backward_vocab_parallel(H, W[a:b].contiguous(), y, lse, a, V, grad_scale=1.0 / N)
        Hr = H.clone().requires_grad_(True)
        Wr = W.clone().requires_grad_(True)
        torch.nn.functional.cross_entropy(Hr @ Wr.T, y).backward()
        q.put((rank, float((dH - Hr.grad).abs().max()), float((dW - Wr.grad[a:b]).abs().max())))
    finally:
        dist.destroy_process_group()


def test_vocab_parallel_backward_allreduce_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_vpb_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    for rank, ddH, ddW in out:
        assert ddH < 1e-12 and ddW < 1e-12


def _bench_vp_worker(rank, world, port, q):
    """bench.vocab_parallel_legs (the `--parallel vocab` step) on two gloo ranks: the
    kernel steps are replaced by fp64 restatements, the exchange and the per-stage
    timing are the benchmark's own."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import linear_cross_entropy_bf16_b200 as flce
        rng = np.random.default_rng(11)
        N, V, D = 7, 13, 5
        H = torch.from_numpy(rng.standard_normal((N, D)))
        W = torch.from_numpy(rng.standard_normal((V, D)))
        y = torch.from_numpy(rng.integers(0, V, N))
        a, b = bench.vocab_shard_bounds(V, world, rank)

        def fake_state(H_, W_shard, y_, v_offset, **kw):
            z = H_ @ W_shard.T
            m = z.max(dim=1).values
            s = torch.exp(z - m[:, None]).sum(dim=1)
            rel = y_ - v_offset
            own = (rel >= 0) & (rel < W_shard.shape[0])
            t = torch.where(own, z[torch.arange(z.shape[0]), rel.clamp(0, W_shard.shape[0] - 1)], 0.0)
            return torch.stack([m, s, t, own.double()], dim=1)

        def fake_merge(states, y_, V_total, **kw):
            m = states[..., 0].max(dim=0).values
            s = (states[..., 1] * torch.exp(states[..., 0] - m)).sum(dim=0)
            lse = m + torch.log(s)
            t = (states[..., 2] * states[..., 3]).sum(dim=0)
            return lse - t, lse, t, (lse - t).mean()

        def fake_shard(H_, W_shard, y_, lse_, v_offset, V_total, grad=None, grad_scale=1.0, **kw):
            p = torch.exp(H_ @ W_shard.T - lse_[:, None])
            rel = y_ - v_offset
            own = (rel >= 0) & (rel < W_shard.shape[0])
            onehot = torch.zeros_like(p)
            onehot[own, rel[own]] = 1.0
            dz = grad_scale * (p - onehot)
            return dz @ W_shard, dz.T @ H_

        flce.shard_state, flce.merge_shards, flce.backward_shard = fake_state, fake_merge, fake_shard
        res = bench.vocab_parallel_legs(flce, H, W[a:b].contiguous(), y, a, V, world, steps=3, warmup=1)
        Hr, Wr = H.clone().requires_grad_(True), W.clone().requires_grad_(True)
        ref = torch.nn.functional.cross_entropy(Hr @ Wr.T, y, reduction="none")
        ref.mean().backward()
        q.put((rank, float((res["loss"] - ref.detach()).abs().max()),
               float((res["dH"] - Hr.grad).abs().max()), float((res["dW_shard"] - Wr.grad[a:b]).abs().max()),
               res["forward"], res["backward"]))
    finally:
        dist.destroy_process_group()


def test_bench_vocab_parallel_legs_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_bench_vp_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    for rank, dloss, ddH, ddW, fw, bw in out:
        assert dloss < 1e-12 and ddH < 1e-12 and ddW < 1e-12
        for key in ("compute_ms", "exchange_ms", "merge_ms", "ms_per_step"):
            assert fw[key] >= 0.0
        assert fw["exchange_bytes_per_rank"] == 16 * 7
        assert bw["ms_per_step"] > 0.0 and bw["exchange_alone_ms"] >= 0.0
        assert bw["exchange_bytes_per_rank"] == 4 * 7 * 5 * 2 * 1 // 2


def test_vocab_shard_bounds_cover_the_vocabulary():
    import bench
    for V, G in [(151936, 8), (13, 2), (5, 4), (1, 1)]:
        bounds = [bench.vocab_shard_bounds(V, G, r) for r in range(G)]
        assert bounds[0][0] == 0 and bounds[-1][1] == V
        assert all(bounds[r][1] == bounds[r + 1][0] for r in range(G - 1))


def test_both_arms_print_the_same_config():
    import bench
    from linear_cross_entropy_bf16_b200 import synth
    w = synth.WORKLOADS[synth.HEADLINE]
    for world in (1, 8):
        for par in ("token", "vocab"):
            assert bench.workload_config(w, world, par) == bench.workload_config(w, world, par)
    c = bench.workload_config(w, 1)
    assert c["workload"] == synth.HEADLINE and c["global_batch"] == 8192 and "no flush" in c["l2"]
    assert "flushed" in bench.workload_config(synth.WORKLOADS["n1024_v32000_d1024"], 1)["l2"]


def test_sustained_summary_bins_chunks_by_clock(tmp_path):
    """The sustained window's clock matching: samples inside each chunk's host time
    span set its clock bin; kernel medians and rates per bin."""
    import bench
    s = bench.ClockSampler(0)
    s.path = str(tmp_path / "c.csv")
    t = 1_700_000_000.0
    with open(s.path, "w") as f:
        for i in range(40):
            ts = datetime_str(t + 0.05 * i)
            mhz = 1900 if i < 20 else 1300
            f.write(f"{ts}, 0, {mhz}, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, "
                    f"{'Active' if i >= 20 else 'Not Active'}\n")
    s.proc, s.f = _Done(), open(os.devnull, "w")
    s.stop()
    assert len(s.rows) == 40
    chunks = [(t, t + 0.9, [1.0, 1.0, 1.2]), (t + 1.0, t + 1.95, [1.5, 1.5, 1.6])]
    peaks = {"bf16_tflops": 1000.0, "bf16_tflops_sustained": 800.0}
    res = bench.sustained_summary(chunks, 1e12, 100, peaks, s)
    assert res["steps"] == 6 and res["kernel_ms_median"] == pytest.approx(1.35)
    assert [b["sm_mhz_bin"] for b in res["by_clock"]] == [1300, 1900]
    assert res["by_clock"][1]["kernel_ms_median"] == pytest.approx(1.0)
    assert res["clocks"]["reasons"] == ["sw_power_cap"]
    assert res["tflops"] == pytest.approx(1e12 / 1.35e-3 / 1e12)


class _Done:
    def terminate(self):
        pass

    def wait(self, *_):
        return 0


def datetime_str(epoch):
    import datetime
    return datetime.datetime.fromtimestamp(epoch).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
