"""The debug build (libgdn_debug.so: the kernels' index checks compiled in) on the GPU,
in a process of its own that loads it through GDN_LIBRARY (tests/debug_build_cases.py).

Every case matches the oracle (1e-2, bf16 I/O) with no failed index check (status 0,
no site); the two calls with GDN_FAULT_BAD_INDEX, whose chains pass one index just past
the record array through the check (nothing is read there), end with GDN_ERR_BAD_INDEX
and a source line, and still match the oracle; the call after them is clean again.
"""
import json
import os
import subprocess
import sys

import pytest

from linear_attention_sequence_delta_b200 import build, gdn
from tests.parity_util import TOL_BF16

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def results():
    path = build.build(debug=True)
    env = dict(os.environ, GDN_LIBRARY=path)
    r = subprocess.run([sys.executable, "-m", "tests.debug_build_cases"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-4000:]
    return {c["case"]: c for c in json.loads(r.stdout.strip().splitlines()[-1])}


CLEAN = ["ragged_half_rows", "ragged_whole_rows", "ragged_split", "many_chains_auto",
         "many_units_split", "slots_padding", "mixer_auto", "mixer_fused", "mixer_split", "after_injection"]


@pytest.mark.parametrize("case", CLEAN)
def test_debug_build_clean(results, case):
    c = results[case]
    assert c["status"] == 0 and c["site"] == 0, c
    assert c["err"] <= TOL_BF16, c


@pytest.mark.parametrize("case", ["inject_split", "inject_overlapped"])
def test_debug_build_reports_injected_index(results, case):
    c = results[case]
    assert c["status"] == 8 and c["site"] > 0, c  # GDN_ERR_BAD_INDEX, a source line
    assert c["err"] <= TOL_BF16, c                # nothing else changed
