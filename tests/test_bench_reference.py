"""The reference arm of bench.py (the float64 oracle on the host cores) on CPU: one JSON line with
the benchmark contract's keys, for the default and the nearest-neighbour workloads; ranks other
than 0 print nothing and exit 0."""

from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                       cwd=ROOT, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return r.stdout


@pytest.mark.parametrize("workload,name", [(None, "large-model-b3"), ("llama", "llama3-8b-decode"),
                                           ("nn-b2", "nn-search-b2")])
def test_reference_arm_line(workload, name):
    # workload None: bench.py's default (the large-model cache at 3 bits)
    out = _run(["--impl", "reference", *(["--workload", workload] if workload else []), "--steps", "1",
                "--warmup", "0"])
    lines = [ln for ln in out.splitlines() if ln.strip()]
    assert len(lines) == 1
    r = json.loads(lines[0])
    assert r["impl"] == "reference" and r["unit"] == "GB/s" and r["value"] > 0
    assert r["higher_is_better"] is True and r["dtype"] == "f64" and r["data"] == "synthetic"
    assert r["config"]["workload"].startswith(name)
    cb = r["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == r["value"] and cb["cores"] >= 1 and cb["sample"]
    assert r["e2e"] == {"value": r["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_are_silent():
    out = _run(["--impl", "reference", "--workload", "nn-b2", "--steps", "1", "--warmup", "0"],
               {"RANK": "1", "WORLD_SIZE": "2"})
    assert out.strip() == ""
