"""gdn_gates (the gate prologue) against the oracle's gates and chunk cumsum."""
import math

import numpy as np
import pytest
import torch

import oracle
from linear_attention_sequence_delta_b200 import gdn_gates
from linear_attention_sequence_delta_b200.inputs import make_prefill_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("lengths", [[256], [1, 63, 64, 65, 127, 0, 300]])
def test_gates_match_oracle(lengths):
    P = make_prefill_inputs(lengths, H_qk=2, H_v=40, d_k=64, d_v=64, seed=5)
    Pd = P.to("cuda")
    G, g, beta = gdn_gates(Pd.a, Pd.b, Pd.A_log, Pd.dt_bias, Pd.cu_seqlens)
    torch.cuda.synchronize()
    g_ref, b_ref = oracle.gates(P.a, P.b, P.A_log, P.dt_bias)
    G_ref = oracle.chunk_cumsum(g_ref, P.cu_seqlens.numpy())
    # fp32 transcendental functions: a few ulp per element, summed over <= 64 terms
    assert np.abs(g.cpu().numpy() - g_ref).max() <= 1e-5 * np.abs(g_ref).max()
    assert np.abs(beta.cpu().numpy() - b_ref).max() <= 1e-6
    assert np.abs(G.cpu().numpy() - G_ref).max() <= 1e-5 * np.abs(G_ref).max()


def test_gates_extremes():
    a = torch.tensor([[-1e30, 0.3, 5.0]], device="cuda")
    b = torch.tensor([[-1e30, 1e30, 0.0]], device="cuda")
    A_log = torch.tensor([0.0, 100.0, 0.0], device="cuda")
    dt = torch.zeros(3, device="cuda")
    cu = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    G, g, beta = gdn_gates(a, b, A_log, dt, cu)
    g = g.cpu()
    assert g[0, 0].item() == 0.0                      # alpha = 1, no NaN
    assert torch.exp(g[0, 1]).item() == 0.0           # alpha = 0 in fp32 (g clamped at -128)
    assert g[0, 1].item() == -128.0
    assert beta.cpu()[0].tolist() == [0.0, 1.0, 0.5]
    assert torch.isfinite(G.cpu()[0, 0])
