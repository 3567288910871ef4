"""Mutation suite: each plausible mistake planted in a copy of the oracle must fail a pin.

Each mutant is a one-line textual change to ``oracle/oracle.cpp`` (a dropped term, a
wrong sign or index, a transposed operand, another rounding). The copy is compiled
into a temporary directory and the whole pin suite runs against it in a child
process (a mutant that reads out of bounds may crash; that also counts as caught).
The unmodified source must pass every pin through the same harness.
"""
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

# (name, old text, new text, which occurrence: 0 = first, None = all)
MUTANTS = [
    ("sign of zero is -1", "if (v < 0.0f) w[c / 32]", "if (v <= 0.0f) w[c / 32]", 0),
    ("bit index transposed", "w[c / 32] |= (1u << (c % 32))", "w[c % 4] |= (1u << (c / 4))", 0),
    ("mu of signed x", "acc += std::fabs(static_cast<double>(p[e]));", "acc += static_cast<double>(p[e]);", 0),
    ("mu over tokens only", "static_cast<float>(acc / cnt)", "static_cast<float>(acc / static_cast<double>(N))", 0),
    ("similarity sign flipped (logits)", "x[(s * N + i) * N + j] = d - 2 * diff;",
     "x[(s * N + i) * N + j] = 2 * diff - d;", 0),
    ("similarity sign flipped (forward)", "const int x = d - 2 * diff;", "const int x = 2 * diff - d;", 0),
    ("similarity uses padded width", "const int x = d - 2 * diff;", "const int x = 128 - 2 * diff;", 0),
    ("V range 128", "const float inv = 127.0f / amax;", "const float inv = 128.0f / amax;", 0),
    ("V truncation", "float r = std::nearbyint(prod);", "float r = std::trunc(prod);", 0),
    ("V scale /255", "sv[s * d + c] = amax / 127.0f;", "sv[s * d + c] = amax / 255.0f;", 0),
    ("bias scaled by alpha", "std::fma(alpha, static_cast<float>(x), bias)",
     "alpha * (static_cast<float>(x) + bias)", 0),
    ("bias dropped", "std::fma(alpha, static_cast<float>(x), bias)", "std::fma(alpha, static_cast<float>(x), 0.0f)", 0),
    ("dense bias transposed", "(h * N + i) * N + j]", "(h * N + j) * N + i]", 0),
    ("relpos offset reversed", "const int64_t row = yi - yj + (bz->table_h - 1);",
     "const int64_t row = yj - yi + (bz->table_h - 1);", 0),
    ("relpos column offset reversed", "const int64_t col = xi - xj + (bz->table_w - 1);",
     "const int64_t col = xj - xi + (bz->table_w - 1);", 0),
    ("relpos row-major on the wrong axis", "const int64_t yi = ti / bz->grid_w, xi = ti % bz->grid_w;",
     "const int64_t yi = ti % bz->grid_h, xi = ti / bz->grid_h;", 0),
    ("class token not exempt", "if (i < bz->n_prefix || j < bz->n_prefix) return 0.0f;",
     "if (i < 0 || j < 0) return 0.0f;", 0),
    ("no rescale of earlier blocks", "std::exp(static_cast<double>(m) - static_cast<double>(mt))", "1.0", 0),
    ("rescale inverted", "std::exp(static_cast<double>(m) - static_cast<double>(mt))",
     "std::exp(static_cast<double>(mt) - static_cast<double>(m))", 0),
    ("P against the stale max", "std::exp(static_cast<double>(s[j - t0]) - static_cast<double>(mt))",
     "std::exp(static_cast<double>(s[j - t0]) - static_cast<double>(m == -std::numeric_limits<float>::infinity() ? mt : m))", 0),
    ("P scale 256", "std::nearbyint(255.0f * p)", "std::nearbyint(256.0f * p)", 0),
    ("P truncation", "std::nearbyint(255.0f * p)", "std::floor(255.0f * p)", 0),
    ("P round half up", "std::nearbyint(255.0f * p)", "std::floor(255.0f * p + 0.5f)", 0),
    ("normaliser from the 8-bit codes", "(a->rowsum_mode == 0) ? static_cast<double>(p)",
     "(a->rowsum_mode != 0) ? static_cast<double>(p)", 0),
    ("output dequantised by 127", "static_cast<double>(sv[bh * d + c2]) / 255.0",
     "static_cast<double>(sv[bh * d + c2]) / 127.0", 0),
    ("V scale of head 0 everywhere", "static_cast<double>(sv[bh * d + c2]) / 255.0",
     "static_cast<double>(sv[c2]) / 255.0", 0),
    ("alpha uses mu_q twice", "(scale * scratch_mu_q[bh]) * scratch_mu_k[bh]",
     "(scale * scratch_mu_q[bh]) * scratch_mu_q[bh]", 0),
    ("default scale 1/d", "1.0f / std::sqrt(static_cast<float>(d))", "1.0f / static_cast<float>(d)", 0),
    ("last key dropped", "const int64_t t1 = (t0 + Bc < N) ? (t0 + Bc) : N;",
     "const int64_t t1 = (t0 + Bc < N) ? (t0 + Bc) : N - 1;", 0),
    ("keys of a block summed twice", "l = l * c + lt;", "l = l * c + 2.0 * lt;", 0),
]

_RUNNER = r"""
import sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import oracle, pins
o = oracle.Oracle({lib!r})
failed = []
for p in pins.ALL_PINS:
    try:
        p(o)
    except Exception as e:
        failed.append(p.__name__)
print("FAILED:" + ",".join(failed))
"""


def _mutate(src: str, old: str, new: str, which):
    assert old in src, f"mutation anchor not found: {old!r}"
    if which is None:
        return src.replace(old, new)
    idx = -1
    for _ in range(which + 1):
        idx = src.index(old, idx + 1)
    return src[:idx] + new + src[idx + len(old):]


def _run_pins(src_text: str, tmp: str, tag: str):
    cpp = os.path.join(tmp, f"m_{tag}.cpp")
    lib = os.path.join(tmp, f"libm_{tag}.so")
    with open(cpp, "w") as f:
        f.write(src_text)
    flags = [f for f in oracle.CXXFLAGS if f != "-O2"] + ["-O1"]
    subprocess.run(["g++", *flags, cpp, "-o", lib], check=True, capture_output=True)
    code = _RUNNER.format(root=ROOT, tests=HERE, lib=lib)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    if r.returncode != 0:
        return None  # crashed: caught
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("FAILED:")][-1]
    return [x for x in line[len("FAILED:"):].split(",") if x]


def test_mutants_are_caught():
    with open(oracle.SOURCE) as f:
        src = f.read()
    with tempfile.TemporaryDirectory() as tmp:
        jobs = [("clean", src)] + [(f"{i}", _mutate(src, old, new, w)) for i, (_, old, new, w) in enumerate(MUTANTS)]
        with ThreadPoolExecutor(max_workers=max(2, (os.cpu_count() or 2))) as ex:
            results = list(ex.map(lambda j: _run_pins(j[1], tmp, j[0]), jobs))
    assert results[0] == [], f"unmodified oracle fails pins through the harness: {results[0]}"
    survivors = [MUTANTS[i][0] for i, r in enumerate(results[1:]) if r == []]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
