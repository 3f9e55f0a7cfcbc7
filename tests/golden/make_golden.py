"""Write tests/golden/oracle_small.txt: a regression fixture for the oracle.

Calls only the oracle and the seeded input generators. Re-run it only when a
change to the oracle's arithmetic is justified by a passage of the pages, and
say which in the commit message.
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from linear_attention_sequence_delta_b200.inputs import make_prefill_inputs  # noqa: E402

SPEC = dict(lengths=[5, 70], H_qk=1, H_v=2, d_k=8, d_v=4, state_std=0.5, seed=3)


def compute():
    import torch
    P = make_prefill_inputs(io_dtype=torch.float32, **SPEC)
    o, Sf = oracle.forward(P.q, P.k, P.v, P.a, P.b, P.A_log, P.dt_bias, P.cu_seqlens.numpy(),
                           P.initial_state)
    return o, Sf


if __name__ == "__main__":
    o, Sf = compute()
    with open(os.path.join(HERE, "oracle_small.txt"), "w") as f:
        f.write("# oracle regression fixture; written by tests/golden/make_golden.py\n")
        f.write(f"# spec {SPEC}\n")
        f.write("o " + " ".join(repr(float(x)) for x in o.ravel()) + "\n")
        f.write("final_state " + " ".join(repr(float(x)) for x in Sf.ravel()) + "\n")
