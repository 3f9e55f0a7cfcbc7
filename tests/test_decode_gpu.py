"""gdn_decode_step against the fp64 oracle (1e-4 fp32 I/O, 1e-2 bf16 I/O)."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_sequence_delta_b200 import gdn_decode_step, gdn_prefill
from linear_attention_sequence_delta_b200.inputs import DECODE_WORKLOAD, make_decode_inputs
from tests.parity_util import TOL_BF16, TOL_FP32, rel_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("io,d", [(torch.float32, 64), (torch.float32, 128),
                                  (torch.bfloat16, 128), (torch.bfloat16, 64)])
def test_decode_steps_match_oracle(io, d):
    steps = 20
    D = make_decode_inputs(steps=steps, num_seqs=6, H_qk=2, H_v=4, d_k=d, d_v=d, io_dtype=io,
                           seed=2)
    state = D.state.cuda()
    S_ref = D.state.numpy().astype(np.float64)
    tol = TOL_FP32 if io == torch.float32 else TOL_BF16
    for t in range(steps):
        o = gdn_decode_step(D.q[t].cuda(), D.k[t].cuda(), D.v[t].cuda(), D.a[t].cuda(),
                            D.b[t].cuda(), D.A_log.cuda(), D.dt_bias.cuda(), state, scale=0.5)
        o_ref, S_ref = oracle.decode_step(D.q[t], D.k[t], D.v[t], D.a[t], D.b[t], D.A_log,
                                          D.dt_bias, S_ref, scale=0.5)
        assert rel_err(o, o_ref) <= tol
    assert rel_err(state, S_ref) <= tol


def test_decode_equals_prefill():
    """T decode steps from a state equal one prefill of T tokens from that state."""
    T = 70
    D = make_decode_inputs(steps=T, num_seqs=1, H_qk=2, H_v=4, d_k=128, d_v=128,
                           io_dtype=torch.float32, seed=4)
    state = D.state.cuda()
    S0 = state.clone()
    os_ = []
    for t in range(T):
        os_.append(gdn_decode_step(D.q[t].cuda(), D.k[t].cuda(), D.v[t].cuda(), D.a[t].cuda(),
                                   D.b[t].cuda(), D.A_log.cuda(), D.dt_bias.cuda(), state))
    cu = torch.tensor([0, T], dtype=torch.int32, device="cuda")
    o, Sf = gdn_prefill(D.q[:, 0].cuda(), D.k[:, 0].cuda(), D.v[:, 0].cuda(), D.a[:, 0].cuda(),
                        D.b[:, 0].cuda(), D.A_log.cuda(), D.dt_bias.cuda(), cu, S0)
    torch.cuda.synchronize()
    assert rel_err(torch.cat(os_), o.cpu().numpy()) <= 1e-5
    assert rel_err(state, Sf.cpu().numpy()) <= 1e-5


def test_decode_workload_1000_steps_sampled():
    """256 sequences x 64 V heads, d=128, bf16, 1000 consecutive in-place steps.
    All 1000 outputs and the final state of 64 of the 256 sequences (every fourth, all
    heads) against the oracle; units are independent, so the sample is exact. The
    oracle runs the 1000 tokens of each sampled sequence as one sequence from its
    initial state, which is the same recurrence (decode steps = prefill, pinned on the
    CPU)."""
    steps = 1000
    D = make_decode_inputs(steps=steps, seed=0, device="cuda", **DECODE_WORKLOAD)
    sample = list(range(0, D.q.shape[1], 4))
    S0 = D.state[sample].cpu()
    state = D.state
    o_all = torch.empty((steps, len(sample), D.v.shape[2], D.v.shape[3]), dtype=D.v.dtype,
                        device="cuda")
    idx = torch.tensor(sample, device="cuda")
    for t in range(steps):
        o = gdn_decode_step(D.q[t], D.k[t], D.v[t], D.a[t], D.b[t], D.A_log, D.dt_bias, state)
        o_all[t] = o.index_select(0, idx)
    torch.cuda.synchronize()
    # groups of 16 sampled sequences packed one after another, steps as tokens
    for g0 in range(0, len(sample), 16):
        grp = sample[g0:g0 + 16]
        pack = lambda x: x[:, grp].transpose(0, 1).reshape(len(grp) * steps,
                                                           *x.shape[2:]).cpu()
        cu = np.arange(len(grp) + 1, dtype=np.int64) * steps
        o_ref, S_ref = oracle.forward(pack(D.q), pack(D.k), pack(D.v), pack(D.a), pack(D.b),
                                      D.A_log.cpu(), D.dt_bias.cpu(), cu, S0[g0:g0 + len(grp)])
        o_ref = o_ref.reshape(len(grp), steps, *o_ref.shape[1:]).transpose(1, 0, 2, 3)
        assert rel_err(o_all[:, g0:g0 + len(grp)], o_ref) <= TOL_BF16, g0
        assert rel_err(state[grp], S_ref) <= TOL_BF16, g0
