"""The oracle pins must catch plausible mistakes in the oracle.

Each mutant is a copy of the oracle's C source with one plausible slip planted in it (a dropped
term, an off-by-one window, a wrong head mapping, ...). It is compiled on the CPU and the pin
suite is run against it; every mutant must make at least one pin fail.
"""
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "sinkattn_oracle.c")

# (name, original text, replacement, occurrence index to replace)
MUTANTS = [
    ("sink dropped from the denominator", "double D = exp(sink - m);", "double D = 0.0;", 0),
    ("sink scaled like a logit", "    double m = sink;\n    for (int j = 0; j < nkeys; ++j) {",
     "    sink = sink * scale;\n    double m = sink;\n    for (int j = 0; j < nkeys; ++j) {", 0),
    ("window one key too wide", "i - window + 1 > 0) ? i - window + 1", "i - window > 0) ? i - window", 0),
    ("causal mask excludes the diagonal", "for (int j = lo; j <= i; ++j)", "for (int j = lo; j < i; ++j)", 0),
    ("GQA head mapping h mod Hkv", "const int g = h / G;", "const int g = h % Hkv;", 0),
    ("LSE in log2", "*lse = m + log(D);", "*lse = m + log2(D);", 0),
    ("weights renormalised without the sink", "double w = exp(a[j] - m) / D;",
     "double w = exp(a[j] - m) / (D - exp(sink - m));", 0),
    ("scale dropped", "a[j] = scale * dot;", "a[j] = dot;", 0),
    ("ring slot off by one", "(ring_head[b] + c) % ring_cap", "(ring_head[b] + c + 1) % ring_cap", 0),
    ("new tokens not causal", "for (int u = 0; u <= t; ++u)", "for (int u = 0; u < T; ++u)", 0),
    ("decode window off by one", "if (p > t || (window > 0 && p <= t - window))",
     "if (p > t || (window > 0 && p < t - window))", 0),
    ("merge counts the sink per span", "D += l_p[p] * exp(m_p[p] - m);",
     "D += l_p[p] * exp(m_p[p] - m) + exp(sink - m);", 0),
    ("paged row ignores the page size", "*\n                                      page_size + c % page_size;",
     "+ c % page_size;", 0),
    ("paged commit takes the page index modulo the page size",
     "row = (int64_t)page_table[(int64_t)b * max_pages + c / page_size] * page_size +\n                      c % page_size;",
     "row = (int64_t)page_table[(int64_t)b * max_pages + c % page_size] * page_size +\n                      c % page_size;", 0),
    ("paged commit ignores the sequence's page-table row",
     "row = (int64_t)page_table[(int64_t)b * max_pages + c / page_size] * page_size +\n                      c % page_size;",
     "row = (int64_t)page_table[c / page_size] * page_size +\n                      c % page_size;", 0),
    ("commit ring overwrites the newest", "slot = ring_head[b];\n", "slot = (ring_head[b] + ring_cap - 1) % ring_cap;\n", 0),
    ("rope sine sign flipped", "yr[i] = a * cs - b * sn;", "yr[i] = a * cs + b * sn;", 0),
    ("rope frequency over the whole head dim", "pow(theta, -2.0 * i / rope_dim)",
     "pow(theta, -2.0 * i / d)", 0),
    ("rope frequency exponent without the 2", "pow(theta, -2.0 * i / rope_dim)",
     "pow(theta, -1.0 * i / rope_dim)", 0),
    ("rope pairs one full width apart", "const int half = rope_dim / 2;", "const int half = rope_dim;", 0),
    ("rope also turns the no-pe dims", "for (int i = 0; i < half; ++i) {\n                const double w",
     "for (int i = 0; i < d / 2; ++i) {\n                const double w", 0),
    ("value scale dropped", "out[e] = bf16_to_f64(v[e]) * v_scale;", "out[e] = bf16_to_f64(v[e]);", 0),
    ("e4m3 ties toward zero", "(d == best_d && (c & 1) == 0)", "(d == best_d && 0)", 0),
    ("e4m3 exponent bias 8", "ldexp((double)(8 + m), e - 10)", "ldexp((double)(8 + m), e - 11)", 0),
    ("e4m3 subnormal step 2^-10", "ldexp((double)m, -9)", "ldexp((double)m, -10)", 0),
    ("e4m3 without saturation", "if (a >= 448.0)\n        return sign | 0x7e;",
     "if (a >= 464.0)\n        return sign | 0x7f;", 0),
    ("fp8 encode multiplies by the scale", "const float y = xi / scale;", "const float y = xi * scale;", 0),
    ("backward drops delta", "const double da = p * (dp[j] - delta);", "const double da = p * dp[j];", 0),
    ("backward sink gradient sign", "gsink[h] += ps * (0.0 - delta);", "gsink[h] += ps * delta;", 0),
    ("backward dk without the scale", "gkj[d] += scale * da * bf16_to_f64(qi[d]);",
     "gkj[d] += da * bf16_to_f64(qi[d]);", 0),
    ("backward dv weighted by da", "gvj[e] += p * bf16_to_f64(di[e]);", "gvj[e] += da * bf16_to_f64(di[e]);", 0),
    ("backward window one key too wide",
     "const int lo = (window > 0 && i - window + 1 > 0) ? i - window + 1 : 0;\n            for (int h = 0; h < Hq; ++h) {\n                const int g = h / G;\n                const double s",
     "const int lo = (window > 0 && i - window > 0) ? i - window : 0;\n            for (int h = 0; h < Hq; ++h) {\n                const int g = h / G;\n                const double s", 0),
]


def _replace_nth(text, old, new, n):
    idx = -1
    for _ in range(n + 1):
        idx = text.find(old, idx + 1)
        assert idx >= 0, f"mutation anchor not found: {old!r}"
    return text[:idx] + new + text[idx + len(old):]


def _run_mutant(tmp, i, name, old, new, n):
    src = open(SRC).read()
    path_c = os.path.join(tmp, f"m{i}.c")
    path_so = os.path.join(tmp, f"m{i}.so")
    open(path_c, "w").write(_replace_nth(src, old, new, n))
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC",
                           "-std=c11", path_c, "-o", path_so, "-lm"])
    env = dict(os.environ, SINKATTN_ORACLE_LIB=path_so, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    return name, r.returncode


def test_every_mutant_is_caught():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            results = list(ex.map(lambda a: _run_mutant(tmp, *a),
                                  [(i,) + m for i, m in enumerate(MUTANTS)]))
    survivors = [name for name, rc in results if rc == 0]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
