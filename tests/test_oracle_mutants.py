"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a temporary copy of oracle/oracle.c (on the CPU, never in the
product), rebuilds that copy and runs the oracle pin tests against it; at least one pin must fail.
"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "e2m1 ties to odd": ("if (a == mid) return (i % 2 == 0) ? i : i + 1;",
                         "if (a == mid) return (i % 2 == 0) ? i + 1 : i;"),
    "ReLU dropped": ("double relu = dot > 0.0 ? dot : 0.0;", "double relu = dot;"),
    "wrong head weight": ("total += (double)w[h] * relu;", "total += (double)w[0] * relu;"),
    "ties to higher index": ("if (a->index < b->index) return -1;",
                             "if (a->index > b->index) return -1;"),
    "nibbles swapped": ("(uint8_t)(c[2 * j] | (c[2 * j + 1] << 4))",
                        "(uint8_t)(c[2 * j + 1] | (c[2 * j] << 4))"),
    "scale divisor": ("float q = amax / 6.0f;", "float q = amax / 5.0f;"),
    "swa scale divisor": ("float s = amax / 448.0f;", "float s = amax / 240.0f;"),
    "block score not max": ("if (items[t].score > m) m = items[t].score;",
                            "if (m == -INFINITY) m = items[t].score;"),
    "pool keeps positions past N": (
        "pool[(int64_t)i * CSA2O_S + r] = (p >= 0 && p < N) ? p : -1;",
        "pool[(int64_t)i * CSA2O_S + r] = p;"),
    "softmax without max shift": ("z[t] = exp(z[t] - m) / l;", "z[t] = exp(z[t]) / l;"),
    "e4m3 bias": ("else v = ldexp(1.0 + (double)m / 8.0, e - 7);",
                  "else v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "negative zero loses sign": ("return (uint8_t)(mag | (f32_signbit(r) ? 8 : 0));",
                                 "return (uint8_t)(mag | (r < 0 ? 8 : 0));"),
    "ring slot off by one": ("int64_t slot = (int64_t)b * W + (p % W);",
                             "int64_t slot = (int64_t)b * W + ((p + 1) % W);"),
    "bf16 rounding ties away from zero": (
        "if (d > 0.5 || (d == 0.5 && fmod(f, 2.0) != 0.0)) r = f + 1.0;",
        "if (d >= 0.5) r = f + 1.0;"),
    "replay window starts one token late": ("int64_t p = (int64_t)N[b] - Wr + r;",
                                            "int64_t p = (int64_t)N[b] - Wr + r + 1;"),
    "replay reads the projection transposed": (
        "acc += (double)bf16_to_f32(hr[k]) * (double)bf16_to_f32(wr[k]);",
        "acc += (double)bf16_to_f32(hr[k]) * (double)bf16_to_f32(w[(int64_t)k * CSA2O_D + j]);"),
    "projection drops the last term": ("      for (int k = 0; k < d; ++k) {\n        double p =",
                                       "      for (int k = 0; k < d - 1; ++k) {\n        double p ="),
    "query/key operands swapped": (
        "dot += (double)bf16_to_f32(iq[h * CSA2O_DI + i]) * (double)bf16_to_f32(k[i]);",
        "dot += (double)bf16_to_f32(iq[i]) * (double)bf16_to_f32(k[h * 0 + i]);"),
    "score tolerance 256x too loose": ("return ldexp(total, -16);", "return ldexp(total, -8);"),
    "score tolerance 256x too tight": ("return ldexp(total, -16);", "return ldexp(total, -24);"),
    "score tolerance drops |w|": ("total += fabs((double)w[h]) * s;", "total += (double)w[h] * s;"),
    "score tolerance sums signed products": (
        "s += fabs((double)bf16_to_f32(iq[h * CSA2O_DI + i]) * (double)bf16_to_f32(k[i]));",
        "s += (double)bf16_to_f32(iq[h * CSA2O_DI + i]) * (double)bf16_to_f32(k[i]);"),
}


def _run(name):
    old, new = MUTANTS[name]
    src = open(os.path.join(ROOT, "oracle", "oracle.c")).read()
    assert old in src, name
    d = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(d, "oracle"),
                        ignore=shutil.ignore_patterns("*.so", "__pycache__"))
        shutil.copytree(os.path.join(ROOT, "tests"), os.path.join(d, "tests"),
                        ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutants.py"))
        with open(os.path.join(d, "oracle", "oracle.c"), "w") as f:
            f.write(src.replace(old, new))
        r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                            "tests/test_oracle_codecs.py", "tests/test_oracle_index_attend.py",
                            "tests/test_oracle_ced.py", "tests/test_oracle_replay.py",
                            "tests/test_oracle_score_tol.py"],
                           cwd=d, capture_output=True, text=True, timeout=600)
        return name, r.returncode
    finally:
        shutil.rmtree(d, ignore_errors=True)


def test_every_planted_mistake_fails_a_pin():
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = dict(ex.map(_run, MUTANTS))
    missed = [n for n, rc in results.items() if rc == 0]
    assert not missed, f"pins did not catch: {missed}"
