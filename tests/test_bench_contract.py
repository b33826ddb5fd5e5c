"""bench.py's output contract, checked on the arm that runs without a GPU.

The reference arm times the oracle on the host cores, so it runs here. It must print one JSON line
with the keys, types and units that the GPU arm's line also carries. The GPU arm itself is covered
by the stack tests, which launch the step the way bench.py times it.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def reference_line():
    env = dict(os.environ)
    env.pop("WORLD_SIZE", None)
    proc = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
         "tiny-full-B1-N4096", "--steps", "2", "--warmup", "1"],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert proc.returncode == 0, proc.stderr[-2000:]
    lines = [ln for ln in proc.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, proc.stdout[-2000:]
    return json.loads(lines[0])


def test_reference_line_has_the_contract_keys(reference_line):
    line = reference_line
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["steps"] == 2 and line["warmup"] == 1 and line["n_gpus"] == 1
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    assert line["vs_baseline"] is None and line["data"] == "synthetic"
    assert line["unit"] == "layer-steps/s" and line["value"] > 0
    assert line["config"]["workload"] == "tiny-full-B1-N4096"


def test_reference_line_baseline_and_e2e(reference_line):
    line = reference_line
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["sample"]
    assert cpu["value"] == line["value"] and cpu["unit"] == line["unit"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    # one layer of B = 1 per step: the step time and the rate agree
    assert abs(line["value"] * line["ms_per_step"] / 1e3 - 1.0) < 0.01
