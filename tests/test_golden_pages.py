"""The page's printed numbers for its production shape (tests/golden/pages_production_shape.json).

The page prints no worked numeric example of the loss itself; what it does
print about the production shape is pinned here, so that the workload
definitions and the benchmark's context figures cannot drift from it.
"""
import json
import math
import os

from linear_cross_entropy_bf16_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_production_shape.json")


def load():
    with open(GOLDEN) as f:
        return json.load(f)


def test_headline_workload_is_the_pages_shape():
    g = load()
    w = synth.WORKLOADS[synth.HEADLINE]
    assert (w.N, w.V, w.D, w.dtype) == (g["N"], g["V"], g["D"], "bf16")


def test_dispatch_count_and_ragged_tail():
    """19 dependent dispatches of 8192 columns cover V = 151936 with a ragged last tile."""
    g = load()
    assert math.ceil(g["V"] / g["vocab_tile_columns"]) == g["dependent_dispatches"]
    assert g["V"] % g["vocab_tile_columns"] == 4480
    # the 256-column tiles used on B200 are ragged too (593 full tiles + 128 columns)
    assert divmod(g["V"], 256) == (593, 128)


def test_printed_slowdown_is_the_ratio_of_printed_times():
    g = load()
    assert round(g["fused_forward_seconds"] / g["materialised_forward_seconds"], 2) == g["fused_over_materialised"]


def test_derived_context_throughput():
    """tokens/s and TFLOP/s that follow from the printed fused time (context for the benchmark)."""
    g = load()
    tok_s = g["N"] / g["fused_forward_seconds"]
    tflops = 2 * g["N"] * g["V"] * g["D"] / g["fused_forward_seconds"] / 1e12
    assert round(tok_s) == 3892
    assert round(tflops, 2) == 4.84
    assert g["max_abs_loss_diff_bf16_inputs"] < 1e-3 and g["max_abs_loss_diff_fp32_inputs"] < 1e-3
