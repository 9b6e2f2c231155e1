"""bench.py --impl reference on the CPU: the oracle arm prints one JSON line
with the contract's keys, on the same metric and workload as the CUDA arm,
its cpu_baseline describing the run and an e2e figure without copies."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e")


@pytest.mark.timeout(300)
@pytest.mark.parametrize("extra", [[], ["--group-agg", "sum"]], ids=["max", "sum"])
def test_reference_arm_json_line(extra):
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1",
                        *extra], cwd=ROOT, capture_output=True, text=True, timeout=280)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for k in KEYS:
        assert k in line, k
    assert line["impl"] == "reference" and line["unit"] == "steps/s" and line["value"] > 0
    assert line["higher_is_better"] is True and line["n_gpus"] == 1 and line["steps"] == 1
    assert line["config"]["workload"].startswith("c128k")
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    # a timed step is a sample of units; ms_per_step is that sample's time and
    # value the whole-step rate it implies
    ss = line["step_sample"]
    frac = ss["units_per_timed_step"] / ss["units_per_decode_step"]
    assert 0 < frac <= 1 and ss["units_per_timed_step"] == cb["cores"]
    assert abs(line["ms_per_step"] - 1e3 * frac / line["value"]) <= 1e-6 * line["ms_per_step"]
