"""The C ABI on the host (no GPU): exports, sizes, schedule and argument checks.

Nothing here launches a kernel: every call below returns before any CUDA API
is reached (argument checks) or is host-only by contract (workspace size,
plan, status strings).
"""
import ctypes
import math
import os
import re

import pytest

import linear_cross_entropy_bf16_b200 as flce
from linear_cross_entropy_bf16_b200 import build as flce_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flce.h")


@pytest.fixture(scope="module")
def lib():
    flce_build.build()
    return flce.load_library()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"FLCE_API\s+[\w\s\*]+?\b(flce_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    assert {"flce_workspace_size", "flce_forward", "flce_check", "flce_status_string",
            "flce_partials", "flce_merge", "flce_plan"} <= names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert getattr(lib, name) is not None


def test_status_strings(lib):
    for s in range(7):
        assert flce.status_string(s) and flce.status_string(s) != "unknown status"
    assert flce.status_string(99) == "unknown status"


def r256(b):
    return (b + 255) // 256 * 256


def state_bytes(N, V):
    """The forward's state: header, one counter per 128-token row block (two per 256
    tokens), the (m, s) partials per (slab, token), one fp64 per 128-token row block."""
    rb = 2 * math.ceil(max(N, 1) / 256)
    slabs = min(math.ceil(V / 256), 512)
    return 256 + r256(4 * rb) + r256(8 * N * slabs) + r256(8 * max(1, math.ceil(N / 128), rb))


def test_workspace_is_O_N_not_O_NV(lib):
    for N, V, D in [(8192, 151936, 4096), (16384, 262144, 2048), (1, 1, 8), (4096, 128256, 4096)]:
        ws = flce.workspace_size(N, V, D)
        slabs = min(math.ceil(V / 256), 512)
        assert ws >= 256 + 8 * N * slabs
        assert ws <= 256 + 8 * N * 512 + 256 + 8 * (N // 32 + 1) + 512 + r256(64 * D)
        if V >= 100000:
            assert ws < 4 * N * V / 50        # the logits it replaces are 4 N V bytes
    assert lib.flce_workspace_size(-1, 10, 8, 0) == 0
    assert lib.flce_workspace_size(4, 0, 8, 0) == 0
    assert lib.flce_workspace_size(4, 10, 0, 0) == 0
    assert lib.flce_workspace_size(4, 10, 8, 7) == 0
    # bf16: the state, independent of D from 32 tokens on; below, plus H padded to
    # 32 rows (32 D bf16)
    assert flce.workspace_size(100, 5000, 64) == flce.workspace_size(100, 5000, 4096)
    for N, V, D in [(100, 5000, 64), (8192, 151936, 4096), (31, 7, 8), (1, 1, 4096), (32, 3, 16)]:
        pad = r256(64 * D) if N < 32 else 0
        assert flce.workspace_size(N, V, D) == state_bytes(N, V) + pad
    # fp32: plus the bf16 hi/lo split copies, H (max(N, 32), 2 Dp) and W (V, 2 Dp), Dp = ceil64(D)
    for N, V, D in [(100, 5000, 64), (256, 2048, 256), (7, 9, 5), (1, 1, 1), (3, 4, 65)]:
        Dp = (D + 63) // 64 * 64
        assert flce.workspace_size(N, V, D, 1) == (state_bytes(N, V) + r256(4 * Dp * max(N, 32))
                                                   + r256(4 * Dp * V))


def unit_order(p):
    """(slab, token block) of each unit, in the documented grouped order."""
    tb, P, gt = p["token_blocks"], p["slabs"], p["group_blocks"]
    order = []
    for g0 in range(0, tb, gt):
        blocks = list(range(g0, min(tb, g0 + gt)))
        order += [(slab, b) for slab in range(P) for b in blocks]
    return order


def simulate_makespan(p):
    base, rem = p["slab_base"], p["slab_rem"]
    workers = p["grid"] // p["ctas_per_unit"]          # CTAs, or CTA pairs
    load = [0] * workers
    for u, (slab, _) in enumerate(unit_order(p)):
        load[u % workers] += base + (1 if slab < rem else 0)
    return max(load)


@pytest.mark.parametrize("N,V,D,dtype,sms", [
    (8192, 151936, 4096, 0, 148), (4096, 128256, 4096, 0, 148), (16384, 262144, 2048, 0, 148),
    (1024, 32000, 1024, 0, 148), (256, 2048, 256, 1, 148), (1, 1, 8, 0, 148), (7, 257, 8, 0, 148),
    (129, 1000, 64, 0, 132), (300, 151936, 128, 0, 148), (2048, 500, 16, 1, 148)])
def test_plan_covers_every_tile_once_and_balances(lib, N, V, D, dtype, sms):
    p = flce.plan(N, V, D, dtype, sm_count=sms)
    assert p["vocab_tiles"] == math.ceil(V / 256)
    assert p["token_blocks"] == math.ceil(N / p["block_rows"])
    assert 1 <= p["slabs"] <= min(p["vocab_tiles"], 512)
    # the slabs partition the vocab tiles
    sizes = [p["slab_base"] + (1 if s < p["slab_rem"] else 0) for s in range(p["slabs"])]
    assert sum(sizes) == p["vocab_tiles"] and min(sizes) >= 1
    assert p["units"] == p["token_blocks"] * p["slabs"]
    order = unit_order(p)
    assert len(order) == p["units"] and len(set(order)) == p["units"]   # each unit exactly once
    assert 1 <= p["group_blocks"] <= p["token_blocks"]
    assert p["workspace_bytes"] == flce.workspace_size(N, V, D, dtype)
    pair = N > 128
    assert p["ctas_per_unit"] == (2 if pair else 1)
    assert p["block_rows"] == (256 if pair else 128)
    workers = sms // 2 if pair else sms
    assert p["grid"] == min(workers, p["units"]) * p["ctas_per_unit"]
    assert simulate_makespan(p) == p["makespan_tiles"]
    total = p["token_blocks"] * p["vocab_tiles"]
    # within one tile per worker of the perfect split, whenever every worker has work;
    # the planner gives up at most 1% of that for slabs of equal length
    if total >= workers:
        bound = math.ceil(total / workers) + 1
        assert p["makespan_tiles"] <= (bound * 1.01 if p["slab_rem"] == 0 else bound)


def test_grouped_makespan_matches_simulation_on_random_shapes(lib):
    import random
    rnd = random.Random(7)
    for _ in range(60):
        N = rnd.choice([rnd.randint(1, 5000), rnd.randint(5000, 70000)])
        V = rnd.randint(1, 300000)
        D = 8 * rnd.randint(1, 1024)
        sms = rnd.choice([148, 132, 120, 16, 2, 1])
        p = flce.plan(N, V, D, 0, sm_count=sms)
        assert simulate_makespan(p) == p["makespan_tiles"], (N, V, D, sms, p)
        order = unit_order(p)
        assert len(set(order)) == p["units"] == len(order)


def test_headline_plan(lib):
    p = flce.plan(8192, 151936, 4096, 0, sm_count=148)
    assert p["ctas_per_unit"] == 2 and p["grid"] == 148
    assert p["block_rows"] == 256 and p["tile_cols"] == 256 and p["k_block"] == 64
    assert p["token_blocks"] == 32 and p["vocab_tiles"] == 594
    assert p["group_blocks"] == 16             # 16 x 2 MB of H live at a time
    assert p["makespan_tiles"] <= 258          # ceil(32 * 594 / 74) = 257 pair tiles
    assert p["slab_rem"] == 0                  # equal slabs (99 x 6 tiles) keep the pairs in step
    # fp32 inputs: the same schedule; the raster group counts only H's hi part
    # (16 blocks, not the 7 that the [hi | lo] rows' bytes would allow)
    q = flce.plan(8192, 151936, 4096, 1, sm_count=148)
    assert q["group_blocks"] == 16 and q["slabs"] == p["slabs"] and q["units"] == p["units"]


def test_plan_rejects_bad_args(lib):
    p = flce.Plan()
    assert lib.flce_plan(4, 10, 8, 0, 0, ctypes.byref(p)) == flce.ERR_INVALID_ARG
    assert lib.flce_plan(-4, 10, 8, 0, 148, ctypes.byref(p)) == flce.ERR_INVALID_ARG
    assert lib.flce_plan(4, 10, 8, 0, 148, None) == flce.ERR_INVALID_ARG


FAKE = 0x10000          # 64 KiB-aligned, never dereferenced: the checks return first


def fwd(lib, H=FAKE, W=FAKE, y=FAKE, N=16, V=100, D=64, dtype=0, loss=FAKE, lse=FAKE, tgt=FAKE,
        mean=None, ws=FAKE, ws_bytes=1 << 30):
    return lib.flce_forward(H, W, y, N, V, D, dtype, loss, lse, tgt, mean, ws, ws_bytes, None)


def test_forward_argument_checks_need_no_gpu(lib):
    assert fwd(lib, N=-1) == flce.ERR_INVALID_ARG
    assert fwd(lib, V=0) == flce.ERR_INVALID_ARG
    assert fwd(lib, D=0) == flce.ERR_INVALID_ARG
    assert fwd(lib, dtype=5) == flce.ERR_INVALID_ARG
    assert fwd(lib, H=None) == flce.ERR_INVALID_ARG
    assert fwd(lib, W=None) == flce.ERR_INVALID_ARG
    assert fwd(lib, y=None) == flce.ERR_INVALID_ARG
    assert fwd(lib, ws=None) == flce.ERR_INVALID_ARG
    assert fwd(lib, loss=None) == flce.ERR_INVALID_ARG
    assert fwd(lib, tgt=None) == flce.ERR_INVALID_ARG
    assert fwd(lib, ws=FAKE + 128) == flce.ERR_INVALID_ARG          # workspace not 256-aligned
    assert fwd(lib, D=60) == flce.ERR_UNSUPPORTED                   # bf16 rows must be 16-byte strided
    assert fwd(lib, H=FAKE + 8) == flce.ERR_UNSUPPORTED             # bf16 base must be 16-byte aligned
    assert fwd(lib, N=1 << 31) == flce.ERR_UNSUPPORTED
    assert fwd(lib, ws_bytes=767) == flce.ERR_WORKSPACE_TOO_SMALL      # needs 768 here
    assert fwd(lib, N=0) == flce.OK                                  # no-op
    assert fwd(lib, N=0, H=None, W=None, y=None, ws=None) == flce.OK


def test_merge_and_partials_argument_checks_need_no_gpu(lib):
    m = lib.flce_merge
    assert m(FAKE, -1, 10, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None) == flce.ERR_INVALID_ARG
    assert m(None, 4, 10, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None) == flce.ERR_INVALID_ARG
    assert m(FAKE, 4, 10, FAKE, FAKE, FAKE, None, FAKE, 10, None) == flce.ERR_WORKSPACE_TOO_SMALL
    assert m(FAKE, 0, 10, None, None, None, None, None, 0, None) == flce.OK
    p = lib.flce_partials
    assert p(FAKE, FAKE, FAKE, 4, 10, 64, 0, None, FAKE, 1 << 30, None) == flce.ERR_INVALID_ARG
    assert p(FAKE, FAKE, FAKE, 4, 10, 64, 0, FAKE, FAKE, 10, None) == flce.ERR_WORKSPACE_TOO_SMALL


def test_selftest_argument_checks_need_no_gpu(lib):
    s = lib.flce_selftest_wait_timeout
    assert s(None, 256, 10000, None) == flce.ERR_INVALID_ARG
    assert s(FAKE, 100, 10000, None) == flce.ERR_INVALID_ARG
    assert s(FAKE, 256, 10, None) == flce.ERR_INVALID_ARG
    assert s(FAKE, 256, 10 ** 10, None) == flce.ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(flce, "_lib", None)
    monkeypatch.setattr(flce, "_LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(flce.FlceError):
        flce.load_library()


def test_forward_ex_argument_checks_need_no_gpu(lib):
    def call(**kw):
        a = dict(H=FAKE, ldh=0, W=FAKE, ldw=0, y=FAKE, y_dtype=0, dtype=0, N=16, V=100, D=64,
                 out_loss=FAKE, out_lse=FAKE, out_target_logit=FAKE, out_mean=None)
        a.update(kw)
        args = flce.ForwardArgs(**a)
        return lib.flce_forward_ex(ctypes.byref(args), kw.get("ws", FAKE), kw.get("ws_bytes", 1 << 30), None)
    assert lib.flce_forward_ex(None, FAKE, 1 << 30, None) == flce.ERR_INVALID_ARG
    assert call(y_dtype=2) == flce.ERR_INVALID_ARG
    assert call(ldh=32) == flce.ERR_INVALID_ARG        # stride below D
    assert call(ldw=65) == flce.ERR_UNSUPPORTED        # bf16 stride not a multiple of 8
    assert call(out_lse=None) == flce.ERR_INVALID_ARG
    assert call(N=0) == flce.OK
    assert call(dtype=1, ldh=65, ldw=66, ws_bytes=10) == flce.ERR_WORKSPACE_TOO_SMALL   # fp32: any stride


def test_quantized_workspace_and_argument_checks_need_no_gpu(lib):
    # size: one chunk's slab state + a float4 per (chunk, token) + one chunk of [hi | lo] rows
    for N, V, D in [(8192, 151936, 4096), (10, 100, 64), (300, 40000, 192)]:
        C = min(V, 16384)
        chunks = math.ceil(V / C)
        Ds = math.ceil(D / 64) * 64
        pad = r256(64 * D) if N < 32 else 0          # H padded with zero rows to 32
        want = state_bytes(N, C) + r256(16 * N * chunks) + r256(C * 2 * Ds * 2) + pad
        assert flce.quantized_workspace_size(N, V, D, 4, 64) == want
    # far below the 4 N V bytes of logits at the page's shape
    assert flce.quantized_workspace_size(8192, 151936, 4096, 4, 64) < 4 * 8192 * 151936 / 10
    for bits, G, D in [(3, 64, 128), (4, 16, 128), (4, 64, 96), (4, 64, 0), (5, 32, 64)]:
        assert lib.flce_quantized_workspace_size(8, 100, D, bits, G) == 0

    def call(bits=4, G=64, N=16, V=100, D=128, H=FAKE, wq=FAKE, s=FAKE, b=FAKE, y=FAKE,
             ws=FAKE, ws_bytes=1 << 30):
        return lib.flce_forward_quantized(H, wq, s, b, bits, G, y, N, V, D, FAKE, FAKE, FAKE, None,
                                          None, ws, ws_bytes, None)
    assert call(bits=3) == flce.ERR_INVALID_ARG
    assert call(G=16) == flce.ERR_INVALID_ARG
    assert call(D=96) == flce.ERR_INVALID_ARG            # not a multiple of G
    assert call(wq=None) == flce.ERR_INVALID_ARG
    assert call(ws=FAKE + 16) == flce.ERR_INVALID_ARG     # workspace must be 256-byte aligned
    assert call(s=FAKE + 1) == flce.ERR_INVALID_ARG       # bf16 scales must be 2-byte aligned
    assert call(H=FAKE + 8) == flce.ERR_UNSUPPORTED       # TMA needs a 16-byte-aligned H
    assert call(wq=FAKE + 4) == flce.ERR_UNSUPPORTED
    assert call(ws_bytes=100) == flce.ERR_WORKSPACE_TOO_SMALL
    assert call(N=0) == flce.OK


def test_forward_host_argument_checks_need_no_gpu(lib):
    for N, V, D in [(300, 20000, 128), (5, 9000, 64)]:
        C = min(V, 8192)
        chunks = math.ceil(V / C)
        want = (state_bytes(N, C) + r256(16 * N * chunks) + r256(max(N, 32) * D * 2) + r256(8 * N)
                + r256(12 * N + 4) + 2 * r256(C * D * 2))
        assert flce.host_workspace_size(N, V, D) == want
    N, V, D = 300, 20000, 128
    assert lib.flce_forward_host_workspace_size(N, V, 12, 0) == 0      # D % 8
    assert lib.flce_forward_host_workspace_size(N, V, D, 1) == 0       # fp32: not supported

    def call(N=16, V=100, D=64, dtype=0, H=FAKE, W=FAKE, y=FAKE, loss=FAKE, ws=FAKE, ws_bytes=1 << 30):
        return lib.flce_forward_host(H, W, y, N, V, D, dtype, loss, None, None, None, ws, ws_bytes,
                                     None, None)
    assert call(H=None) == flce.ERR_INVALID_ARG
    assert call(loss=None) == flce.ERR_INVALID_ARG
    assert call(ws=FAKE + 64) == flce.ERR_INVALID_ARG
    assert call(dtype=1) == flce.ERR_UNSUPPORTED
    assert call(D=12) == flce.ERR_UNSUPPORTED
    assert call(ws_bytes=1000) == flce.ERR_WORKSPACE_TOO_SMALL
    assert call(N=0) == flce.OK


def test_backward_workspace_fp32_adds_split_copies(lib):
    r256 = lambda b: (b + 255) // 256 * 256
    for N, V, D in [(8192, 151936, 4096), (7, 3, 5), (300, 40000, 96)]:
        chunk = min(math.ceil(V / 256) * 256, 32768)       # bf16
        chunk32 = min(math.ceil(V / 256) * 256, 16384)     # fp32
        Dp = (D + 7) // 8 * 8
        if D % 8 == 0:
            assert flce.backward_workspace_size(N, V, D) == 256 + r256(2 * N * chunk)
        assert flce.backward_workspace_size(N, V, D, 1) == (
            256 + 2 * r256(2 * N * chunk32) + r256(6 * Dp * N) + r256(6 * Dp * chunk32))


def test_quantized_backward_workspace_and_checks_need_no_gpu(lib):
    r256 = lambda b: (b + 255) // 256 * 256
    N, V, D = 300, 40000, 96
    chunk = 16384
    Ds = 128
    assert flce.backward_quantized_workspace_size(N, V, D, 4, 32) == 256 + r256(2 * N * chunk) + r256(chunk * 2 * Ds * 2)
    assert lib.flce_backward_quantized_workspace_size(N, V, D, 4, 64) == 0     # 96 % 64 != 0

    def call(bits=4, G=64, N=16, V=100, D=128, H=FAKE, lse=FAKE, dH=FAKE, ws=FAKE, ws_bytes=1 << 30):
        return lib.flce_backward_quantized(H, FAKE, FAKE, FAKE, bits, G, FAKE, lse, None, 1.0, N, V, D,
                                           dH, ws, ws_bytes, None)
    assert call(bits=3) == flce.ERR_INVALID_ARG
    assert call(lse=None) == flce.ERR_INVALID_ARG
    assert call(dH=None) == flce.ERR_INVALID_ARG
    assert call(H=FAKE + 8) == flce.ERR_UNSUPPORTED
    assert call(ws_bytes=64) == flce.ERR_WORKSPACE_TOO_SMALL
    assert call(N=0) == flce.OK


def test_backward_shard_checks_need_no_gpu(lib):
    def call(V_shard=100, v_offset=0, V_total=1000, N=16):
        return lib.flce_backward_shard(FAKE, FAKE, FAKE, FAKE, None, 1.0, N, V_shard, v_offset, V_total,
                                       64, 0, FAKE, FAKE, FAKE, 1 << 30, None, None)
    assert call(v_offset=-1) == flce.ERR_INVALID_ARG
    assert call(v_offset=950) == flce.ERR_INVALID_ARG        # shard runs past V_total
    assert call(V_shard=0) == flce.ERR_INVALID_ARG
    assert call(N=0) == flce.OK


# ---- the partition-aware order of the pair kernel (host-only queries) ----

def partition_lists(lib, TB, P, u0):
    out = (ctypes.c_int32 * (2 * TB * P))()
    assert lib.flce_partition_order(TB, P, u0, out) == flce.OK
    units = [(out[2 * i], out[2 * i + 1]) for i in range(TB * P)]
    return units[:u0], units[u0:]


@pytest.mark.parametrize("TB,P,u0", [
    (32, 99, 1584), (32, 99, 1498), (32, 99, 1), (32, 99, 98), (32, 99, 99), (32, 99, 3167),
    (2, 3, 1), (2, 3, 3), (2, 3, 5), (1, 7, 4), (64, 128, 4027), (17, 5, 0), (17, 5, 85)])
def test_partition_order_covers_every_unit_once(lib, TB, P, u0):
    side0, side1 = partition_lists(lib, TB, P, u0)
    assert sorted(side0 + side1) == [(p, t) for p in range(P) for t in range(TB)]
    q, r = divmod(u0, P)
    # partition 0: token blocks [0, q) and slabs [0, r) of block q; partition 1 the rest
    assert set(side0) == {(p, t) for p in range(P) for t in range(TB)
                          if t < q or (t == q and p < r)}
    # each side walks its units slab by slab
    for units in (side0, side1):
        slabs = [p for p, _ in units]
        assert slabs == sorted(slabs)
        for p in set(slabs):
            blocks = [t for s, t in units if s == p]
            assert blocks == sorted(blocks)


def test_partition_order_rejects_bad_arguments(lib):
    out = (ctypes.c_int32 * 64)()
    for args in ((0, 4, 0), (4, 0, 0), (4, 4, -1), (4, 4, 17)):
        assert lib.flce_partition_order(*args, out) == flce.ERR_INVALID_ARG
    assert lib.flce_partition_order(4, 4, 3, None) == flce.ERR_INVALID_ARG


@pytest.mark.parametrize("n0,n1", [(37, 37), (35, 39), (1, 5), (5, 1), (2, 2)])
def test_partition_take_gives_every_rank_once_however_pairs_land(lib, n0, n1):
    """Whatever number a0 of the n0 + n1 pairs lands on partition 0, the pairs'
    (partition, rank) are exactly the planned ones."""
    s, r = ctypes.c_int32(), ctypes.c_int32()
    for a0 in range(n0 + n1 + 1):
        taken = []
        for side, count in ((0, a0), (1, n0 + n1 - a0)):
            for arrival in range(count):
                assert lib.flce_partition_take(n0, n1, side, arrival, ctypes.byref(s),
                                               ctypes.byref(r)) == flce.OK
                taken.append((s.value, r.value))
        assert sorted(taken) == [(0, k) for k in range(n0)] + [(1, k) for k in range(n1)]


def test_partition_take_rejects_bad_arguments(lib):
    s, r = ctypes.c_int32(), ctypes.c_int32()
    for args in ((0, 3, 0, 0), (3, 0, 0, 0), (3, 3, 2, 0), (3, 3, 0, 6), (3, 3, 0, -1)):
        assert lib.flce_partition_take(*args, ctypes.byref(s), ctypes.byref(r)) == flce.ERR_INVALID_ARG
    assert lib.flce_partition_take(3, 3, 0, 0, None, ctypes.byref(r)) == flce.ERR_INVALID_ARG


def test_partition_map_rejects_null(lib):
    assert lib.flce_partition_map(None) == flce.ERR_INVALID_ARG
