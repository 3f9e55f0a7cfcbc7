"""Fixtures under tests/golden: the pages' printed sizes, and the oracle regression file."""
import os

import numpy as np

from linear_attention_sequence_delta_b200 import inputs
from tests.golden import make_golden

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _sizes():
    out = {}
    for line in open(os.path.join(GOLD, "qwen35_gdn_sizes.txt")):
        if line.startswith("#") or not line.strip():
            continue
        name, val = line.split()[:2]
        out[name] = float(val)
    return out


def test_workloads_use_the_pages_shapes():
    s = _sizes()
    w35 = inputs.WORKLOADS["prefill_35b"]
    assert (w35["H_qk"], w35["H_v"]) == (s["linear_num_key_heads"], s["linear_num_value_heads"])
    assert (w35["d_k"], w35["d_v"]) == (s["head_k_dim"], s["head_v_dim"])
    w397 = inputs.WORKLOADS["prefill_397b_long"]
    assert (w397["H_qk"], w397["H_v"]) == (s["qk_heads_397b"], s["value_heads_397b"])
    assert inputs.DECODE_WORKLOAD["H_v"] == s["value_heads_397b"]


def test_state_size_matches_the_pages_figure():
    s = _sizes()
    per_layer = s["linear_num_value_heads"] * s["head_k_dim"] * s["head_v_dim"] * 4  # fp32
    total_mb = s["gdn_layers_35b"] * per_layer / 1e6
    assert round(total_mb, 1) == s["gdn_state_mb_30_layers"]


def test_oracle_regression_fixture():
    lines = {ln.split()[0]: ln.split()[1:] for ln in open(os.path.join(GOLD, "oracle_small.txt"))
             if not ln.startswith("#")}
    o, Sf = make_golden.compute()
    assert np.abs(o.ravel() - np.array(lines["o"], dtype=float)).max() < 1e-12
    assert np.abs(Sf.ravel() - np.array(lines["final_state"], dtype=float)).max() < 1e-12
