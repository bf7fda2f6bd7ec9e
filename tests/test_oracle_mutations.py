"""Plant plausible mistakes in copies of the oracle and check that the pins
catch every one (CPU only).

Each mutant is the oracle's source with one textual change, compiled into a
temporary directory and exercised in a child process, so a mutant can never
touch the real oracle or crash the test process.
"""
import concurrent.futures as cf
import os
import subprocess
import sys
import tempfile

import pytest

from oracle import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (name, text in oracle.cpp, replacement)
MUTANTS = [
    ("bias is the max", "float bias = mn;", "float bias = mx;"),
    ("range drops min", "float range = mx - mn;", "float range = mx;"),
    ("2^b levels", "const float levels = (float)((1u << bits) - 1u);",
     "const float levels = (float)(1u << bits);"),
    ("round half away", "std::nearbyint(t)", "std::round(t)"),
    ("truncate", "std::nearbyint(t)", "std::trunc(t)"),
    ("pack reversed", "codes[wi] |= q << (j * bits);",
     "codes[wi] |= q << ((per_word - 1 - j) * bits);"),
    ("unpack reversed", "return (word >> (j * bits)) & ((1u << bits) - 1u);",
     "return (word >> ((per_word - 1 - j) * bits)) & ((1u << bits) - 1u);"),
    ("bias dropped", "return s * (double)code_at(codes, row, col, cols, bits) + b;",
     "return s * (double)code_at(codes, row, col, cols, bits);"),
    ("bias sign", "return s * (double)code_at(codes, row, col, cols, bits) + b;",
     "return s * (double)code_at(codes, row, col, cols, bits) - b;"),
    ("wrong group index", "int64_t g = row * (cols / gs) + col / gs;",
     "int64_t g = row * (cols / gs) + (col / gs) / 2;"),
    ("transposed operand", ": dequant_at(codes, scales, biases, sdtype, k, n, N, gs, bits);",
     ": dequant_at(codes, scales, biases, sdtype, n, k, K, gs, bits);"),
    ("magnitude signed", "mag += std::fabs(p);", "mag += p;"),
    ("bf16 ties away", "if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u))) keep += 1;",
     "if (rest >= 0x8000u) keep += 1;"),
    ("bf16 truncates", "if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u))) keep += 1;",
     "(void)rest;"),
    ("gather wrong expert", "        int64_t e = (int64_t)rhs[r];\n            dot_one",
     "        int64_t e = (int64_t)rhs[R - 1 - r];\n            dot_one"),
    ("signed zero by order", "if (v < mn || (v == mn && std::signbit(v))) mn = v;",
     "if (v < mn) mn = v;"),
    ("constant group top code", "uint32_t q = 0;", "uint32_t q = (uint32_t)levels;"),
    ("gather_mm wrong expert", "const int64_t wrow = ((int64_t)rhs[r] * N + n) * K;",
     "const int64_t wrow = ((int64_t)rhs[R - 1 - r] * N + n) * K;"),
    ("gather_mm ignores lhs", "const int64_t t = lhs ? (int64_t)lhs[r] : r;",
     "const int64_t t = r % x_rows;"),
    ("gather_mm transposed expert", "load_value(w, wdtype, wrow + k)",
     "load_value(w, wdtype, (int64_t)rhs[r] * N * K + k * N + n)"),
    ("silu sign", "h[i] = g / (1.0 + std::exp(-g)) * u;", "h[i] = g / (1.0 + std::exp(g)) * u;"),
    ("gate and up swapped", "h[i] = g / (1.0 + std::exp(-g)) * u;",
     "h[i] = u / (1.0 + std::exp(-u)) * g;"),
    ("routing weight dropped", "yt[n] += w * acc;", "yt[n] += acc;"),
    ("stored value rounded through fp32",
     "const double v = round_to_odd_sum(p, load_value(biases, sdtype, g));",
     "const double v = (double)(float)(p + load_value(biases, sdtype, g));"),
    ("stored value rounded through fp64", "if (err == 0.0 || !std::isfinite(sum)) return sum;",
     "return sum;"),
    ("tolerance drops the gate term", "std::fabs(dsilu * u) * ag", "0.0 * ag"),
    ("tolerance drops the up term", "std::fabs(g * sg) * au", "0.0 * au"),
    ("tolerance silu slope", "const double dsilu = sg * (1.0 + g * (1.0 - sg));",
     "const double dsilu = sg;"),
    ("out-of-range expert kept", "const int64_t e = (int64_t)ids[t * topk + j];",
     "const int64_t e = (int64_t)ids[t * topk + j] % E;"),
    ("down transposed", "dequant_at(dc, dsc, dbi, sdtype, n, i, I, gs, bits)",
     "dequant_at(dc, dsc, dbi, sdtype, i, n, K, gs, bits)"),
    ("e2m1 exponent bias", "std::ldexp(1.0 + 0.5 * m, e - 1)", "std::ldexp(1.0 + 0.5 * m, e - 2)"),
    ("e4m3 exponent bias", "std::ldexp(1.0 + m / 8.0, e - 7)", "std::ldexp(1.0 + m / 8.0, e - 8)"),
    ("e8m0 bias", "std::ldexp(1.0, (int)c - 127)", "std::ldexp(1.0, (int)c - 128)"),
    ("fp ties to larger", "(d == best_d && (c & 1u) == 0u)", "(d == best_d)"),
    ("fp no saturation", "if (a >= gmax) best = top;", "(void)gmax;"),
    ("fp sign dropped", "return std::signbit(v) ? (best | sign_bit) : best;", "return best;"),
    ("mx scale rounds up", "const int e = (ex - 1) - (elem == 0 ? 2 : 8);",
     "const int e = ex - (elem == 0 ? 2 : 8);"),
    ("nvfp4 scale over 4", "const float sv = amax / 6.0f;", "const float sv = amax / 4.0f;"),
    ("fp scale index", "scales[row * (cols / gs) + col / gs]", "scales[row * (cols / gs) + col / (2 * gs)]"),
]

RUNNER = r"""
import sys
sys.path.insert(0, {root!r})
import oracle as O
from tests import oracle_pins as P
lib = O.load({lib!r})
failed = []
for pin in P.ALL_PINS:
    try:
        pin(lib)
    except Exception as e:
        failed.append(pin.__name__)
print(",".join(failed))
sys.exit(1 if failed else 0)
"""


def _run_mutant(args):
    name, old, new, tmp = args
    src = open(B.SRC).read()
    assert src.count(old) >= 1, f"mutation site not found: {name}"
    mutated = src.replace(old, new, 1)
    d = os.path.join(tmp, name.replace(" ", "_"))
    os.makedirs(d)
    cpp = os.path.join(d, "oracle.cpp")
    lib = os.path.join(d, "liboracle.so")
    with open(cpp, "w") as f:
        f.write(mutated)
    B.build(cpp, lib, extra=["-O1"])
    r = subprocess.run([sys.executable, "-c", RUNNER.format(root=ROOT, lib=lib)],
                       capture_output=True, text=True, timeout=300,
                       env={**os.environ, "OMP_NUM_THREADS": "1"})
    return name, r.returncode, r.stdout.strip(), r.stderr[-400:]


def test_every_mutant_is_caught():
    with tempfile.TemporaryDirectory() as tmp:
        jobs = [(n, o, w, tmp) for n, o, w in MUTANTS]
        with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            results = list(ex.map(_run_mutant, jobs))
    survivors = [(n, out, err) for n, rc, out, err in results if rc == 0]
    assert not survivors, f"mutants not caught by any pin: {survivors}"


def test_unmutated_copy_passes():
    """Control: the unchanged source, built the same way, passes every pin."""
    with tempfile.TemporaryDirectory() as tmp:
        name, rc, out, err = _run_mutant(("control", "float bias = mn;", "float bias = mn;", tmp))
    assert rc == 0, (out, err)
