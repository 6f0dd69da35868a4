"""A plain C program (tests/c_abi/flce_from_c.c) calls the forward through
include/flce.h and libflce.so alone: no Python binding, no torch on its side.

On the CPU the program compiles and links with gcc against the header and the
library (the boundary is usable from C as declared).  On the GPU it runs on
seeded inputs written to files, and every row it writes matches the oracle.
"""
import os
import subprocess

import numpy as np
import pytest

from linear_cross_entropy_bf16_b200 import build as flce_build
from linear_cross_entropy_bf16_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi", "flce_from_c.c")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def compile_program(out_dir):
    lib = flce_build.build()
    exe = os.path.join(str(out_dir), "flce_from_c")
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c11", "-O1", "-Wall", "-Werror", SRC, "-o", exe,
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           "-L", libdir, "-l:libflce.so", f"-Wl,-rpath,{libdir}",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


def test_program_compiles_against_header_and_library(tmp_path):
    exe = compile_program(tmp_path)
    assert os.access(exe, os.X_OK)


@pytest.mark.gpu
@pytest.mark.parametrize("N,V,D", [(300, 5000, 128), (129, 70001, 72)])
def test_program_output_matches_oracle(tmp_path, N, V, D):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import oracle
    from tests.flce_testing import compare
    oracle.build()
    exe = compile_program(tmp_path)
    H, W, y = synth.random_inputs(N, V, D, seed=N + V)
    paths = {k: os.path.join(str(tmp_path), f"{k}.bin") for k in ("H", "W", "y", "out")}
    np.ascontiguousarray(H).tofile(paths["H"])
    np.ascontiguousarray(W).tofile(paths["W"])
    np.ascontiguousarray(y, dtype=np.int64).tofile(paths["y"])
    r = subprocess.run([exe, str(N), str(V), str(D), paths["H"], paths["W"], paths["y"], paths["out"]],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    out = np.fromfile(paths["out"], dtype=np.float32).astype(np.float64)
    assert out.size == 3 * N + 1
    gpu = {"loss": out[:N], "lse": out[N:2 * N], "target": out[2 * N:3 * N], "mean": float(out[3 * N])}
    ref = oracle.forward(H, W, y)
    compare(gpu, ref, mean_ref=oracle.mean(ref["loss"]))
