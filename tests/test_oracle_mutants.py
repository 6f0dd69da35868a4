"""The oracle's pins catch planted mistakes (CPU only).

Each mutant is a copy of oracle/oracle.c with one plausible mistake planted
(a dropped term, a wrong sign, a wrong index, a swapped operand order, a
wrong base or shift), compiled with gcc into a temporary shared object.  The
CPU pin suites then run against it in a subprocess (ORACLE_LIB_PATH points
the oracle module at the mutant) and must fail.  The unmutated source,
compiled the same way, must pass: the harness itself is sound.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

FWD = ["tests/test_oracle_pins.py", "tests/test_golden_pages.py"]
BWD = ["tests/test_oracle_backward_pins.py"]
QNT = ["tests/test_oracle_quant_pins.py"]

FR = "int oracle_forward_rows("
QR = "int oracle_forward_quantized_rows("
BW = "int oracle_backward("
WR = "int oracle_grad_weight_rows("

# (name, text in oracle.c, replacement, which occurrence of the text, pin files
# that cover the mutated function, the function the mutation must land in)
MUTANTS = [
    ("lse drops the max shift", "double lse = M + log(S);", "double lse = log(S);", 0, FWD, FR),
    ("loss sign flipped", "out_loss[t] = lse - tgt;", "out_loss[t] = tgt - lse;", 0, FWD, FR),
    ("target logit off by one column", "double tgt = z[y[i]];",
     "double tgt = z[y[i] > 0 ? y[i] - 1 : 0];", 0, FWD, FR),
    ("logit pairs H_ik with W_j,D-1-k", "load_elem(W, dtype, j * D + k)",
     "load_elem(W, dtype, j * D + (D - 1 - k))", 0, FWD, "static double logit("),
    ("sum of exponentials drops column 0", "for (int64_t j = 0; j < V; ++j) S += exp(z[j] - M);",
     "for (int64_t j = 1; j < V; ++j) S += exp(z[j] - M);", 0, FWD, FR),
    ("exp taken base 2", "S += exp(z[j] - M);", "S += exp2(z[j] - M);", 0, FWD, FR),
    ("bf16 widened by 15 bits", "((const uint16_t *)base)[idx]) << 16;",
     "((const uint16_t *)base)[idx]) << 15;", 0, FWD, "static double load_elem("),
    ("mean divides by n - 1", "return acc / (double)n;", "return acc / (double)(n - 1);", 0, FWD,
     "double oracle_mean("),
    ("backward one-hot sign flipped", "(exp(z[j] - lse[i]) - (j == y[i] ? 1.0 : 0.0))",
     "(exp(z[j] - lse[i]) + (j == y[i] ? 1.0 : 0.0))", 0, BWD, BW),
    ("backward dH drops the W factor", "acc += z[j] * w;", "acc += z[j];", 0, BWD, BW),
    ("backward dW drops the H factor", "acc += dz[i] * h;", "acc += dz[i];", 0, BWD, BW),
    ("dW row sampler flips the one-hot sign", "(exp(logit(H, W, dtype, i, j, D) - lse[i]) -\n"
     "                                    (j == y[i] ? 1.0 : 0.0));",
     "(exp(logit(H, W, dtype, i, j, D) - lse[i]) +\n"
     "                                    (j == y[i] ? 1.0 : 0.0));", 1, BWD, WR),
    ("dW row sampler's lse drops the max shift", "lse[i] = M + log(S);", "lse[i] = log(S);", 1, BWD, WR),
    ("dW row sampler pairs dZ with the wrong token", "acc += dz[i] * h;",
     "acc += dz[N - 1 - i] * h;", 1, BWD, WR),
    ("quantised codes read highest first", "(word >> (bits * (int)(k % per_word)))",
     "(word >> (bits * (int)(per_word - 1 - k % per_word)))", 0, QNT, "static uint32_t quant_code("),
    ("quantised groups in reverse order", "const int64_t g = j * (D / G) + k / G;",
     "const int64_t g = j * (D / G) + (D / G - 1 - k / G);", 0, QNT, "static double dequant_elem("),
    ("quantised bias dropped", "bf16_bits_value(biases[g]);", "0.0 * bf16_bits_value(biases[g]);",
     0, QNT, "static double dequant_elem("),
    ("quantised lse drops the max shift", "double lse = M + log(S);", "double lse = log(S);", 3, QNT, QR),
    ("quantised target logit off by one column", "double tgt = z[y[i]];",
     "double tgt = z[y[i] > 0 ? y[i] - 1 : 0];", 1, QNT, QR),
    ("quantised logit skips the last element",
     "for (int64_t k = 0; k < D; ++k)\n                    acc += h[k] * dequant_elem",
     "for (int64_t k = 0; k < D - 1; ++k)\n                    acc += h[k] * dequant_elem", 0, QNT, QR),
]


def lands_in(text, pos, header):
    """The mutation at `pos` lies inside the body of the function whose definition
    starts with `header` (no function end between that header and `pos`)."""
    start = text.rfind(header, 0, pos)
    return start >= 0 and text.find("\n}\n", start, pos) < 0


def build_variant(tmp_path, name, text):
    src = tmp_path / f"{name}.c"
    src.write_text(text)
    lib = tmp_path / f"{name}.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(lib),
                           str(src), "-lm"])
    return str(lib)


def run_pins(lib, pins, stop_first=True):
    env = dict(os.environ, ORACLE_LIB_PATH=lib, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "not gpu"] + pins
    if stop_first:
        cmd.insert(3, "-x")
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_unmutated_oracle_passes_the_pins(tmp_path):
    r = run_pins(build_variant(tmp_path, "original", open(SRC).read()), FWD + BWD + QNT,
                 stop_first=False)
    assert r.returncode == 0, r.stdout[-2000:]


def test_pins_catch_every_planted_mistake(tmp_path):
    text = open(SRC).read()
    jobs = []
    for n, (name, old, new, occurrence, pins, fn) in enumerate(MUTANTS):
        parts = text.split(old)
        assert len(parts) > occurrence + 1, f"mutation target not found: {old!r}"
        pos = len(old.join(parts[:occurrence + 1]))
        assert lands_in(text, pos, fn), f"mutant '{name}' does not land in {fn}"
        mutated = old.join(parts[:occurrence + 1]) + new + old.join(parts[occurrence + 1:])
        assert mutated != text
        jobs.append((name, build_variant(tmp_path, f"mutant{n}", mutated), pins))
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with ThreadPoolExecutor(workers) as ex:
        results = list(ex.map(lambda j: (j[0], run_pins(j[1], j[2])), jobs))
    survivors = [name for name, r in results
                 if r.returncode == 0 or not ("failed" in r.stdout or "error" in r.stdout.lower())]
    assert not survivors, f"no pin caught: {survivors}"
