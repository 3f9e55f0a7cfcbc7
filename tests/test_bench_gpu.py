"""bench.py's JSON line on a small invocation (the headline workload restricted to its
first eight sequences, one timed step): one line with the contract's keys, the roofline of
the dominant kernel, the launch count of the library's kernels and the run's metadata."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_contract():
    cmd = [sys.executable, "bench.py", "--steps", "1", "--warmup", "3", "--seqs", "8",
           "--no-decode", "--no-mixer", "--no-other-prefill", "--no-e2e", "--no-cpu-baseline"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-4000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "gpu_launches", "clocks", "run"):
        assert key in line, key
    assert line["value"] > 0 and line["steps"] == 1 and line["n_gpus"] == 1
    roof = line["roofline"]
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    assert 0 < roof["frac"] == pytest.approx(roof["achieved"] / roof["peak"])
    assert line["gpu_launches"] == 3  # chunk offsets, preparation, chains
    run = line["run"]
    assert run["gpu"]["name"] and run["gpu"]["sm_count"] > 0
    assert len(run["library"]["sources_sha1"]) == 40 and run["library"]["debug_build"] is False
