"""gdn_decode_step_bf16_state against the fp64 oracle, and the tolerance study of the
bf16 state ("Qwen3.5-MoE-35B-A3B architecture teardown", section 9.4).

Every step rounds the state to bf16, a relative error of at most u = 2^-9 per entry.
The oracle starts from the same bf16-rounded state (read exactly) and keeps fp64 from
there, so the gap is the accumulated rounding: after one step it is about u of the
state's scale; over many steps each earlier rounding is multiplied by the later decays
and (I - beta k k^T) contractions, so it stays near u / (1 - alpha) in the worst case and
near u / sqrt(1 - alpha^2) for independent roundings. The bars below follow from that:
one step 1e-2 (the bf16 I/O bar); 300 steps with the workload's gates (alpha mostly
well below 0.9) 1e-2; 300 steps of slow decay (alpha ~ 0.987, worst-case growth ~77 u,
independent-rounding estimate ~6 u) 3e-2. The measured values are printed.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_sequence_delta_b200 import (gdn_decode_step, gdn_decode_step_bf16_state,
                                                  gdn_sync_status)
from linear_attention_sequence_delta_b200.inputs import make_decode_inputs
from tests.parity_util import TOL_BF16, rel_err

pytestmark = pytest.mark.gpu


def _run(D, steps, bf16_state):
    st = D.state.to(torch.bfloat16)  # both runs start from the bf16-rounded state
    st = st if bf16_state else st.float()
    st = st.cuda()
    q, k, v, a, b = (x.cuda() for x in (D.q, D.k, D.v, D.a, D.b))
    A_log, dt_bias = D.A_log.cuda(), D.dt_bias.cuda()
    os_ = []
    for t in range(steps):
        f = gdn_decode_step_bf16_state if bf16_state else gdn_decode_step
        os_.append(f(q[t], k[t], v[t], a[t], b[t], A_log, dt_bias, st))
    assert gdn_sync_status() == 0
    return torch.stack(os_), st


def _oracle(D, steps, S0):
    """The steps of each sequence as one packed run (decode = prefill is pinned)."""
    N = D.q.shape[1]
    seq = lambda x: x[:steps].transpose(0, 1).reshape(N * steps, *x.shape[2:])
    cu = np.arange(N + 1) * steps
    o, S = oracle.forward(seq(D.q), seq(D.k), seq(D.v), seq(D.a), seq(D.b), D.A_log,
                          D.dt_bias, cu, S0)
    return o.reshape(N, steps, *o.shape[1:]).transpose(1, 0, 2, 3), S


def test_one_step_bf16_state():
    D = make_decode_inputs(steps=1, num_seqs=16, H_qk=4, H_v=8, d_k=128, d_v=128, seed=1)
    o, st = _run(D, 1, True)
    o_ref, S_ref = _oracle(D, 1, D.state.to(torch.bfloat16))
    assert rel_err(o, o_ref) <= TOL_BF16 and rel_err(st, S_ref) <= TOL_BF16


@pytest.mark.parametrize("regime,bar", [("workload", 1e-2), ("slow_decay", 3e-2)])
def test_bf16_state_drift_over_300_steps(regime, bar):
    steps = 300
    D = make_decode_inputs(steps=steps, num_seqs=4, H_qk=2, H_v=4, d_k=128, d_v=128, seed=2)
    if regime == "slow_decay":
        D.A_log.fill_(-4.0)
    o16, s16 = _run(D, steps, True)
    o32, s32 = _run(D, steps, False)
    S0 = D.state.to(torch.bfloat16)
    o_ref, S_ref = _oracle(D, steps, S0)
    e16 = [rel_err(o16[t], o_ref[t]) for t in (0, 9, 99, steps - 1)]
    e32 = [rel_err(o32[t], o_ref[t]) for t in (0, 9, 99, steps - 1)]
    es16, es32 = rel_err(s16, S_ref), rel_err(s32, S_ref)
    print(f"\n{regime}: o err at steps 1/10/100/{steps}: bf16 state {e16}, fp32 state {e32}; "
          f"final state err: bf16 {es16:.3e}, fp32 {es32:.3e}")
    assert max(e16) <= bar and es16 <= bar
