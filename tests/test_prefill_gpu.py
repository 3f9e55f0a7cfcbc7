"""gdn_prefill (gate prologue + chunk kernel) against the fp64 oracle.

Tolerance (max|gpu - oracle| / max|oracle|, on o and on the final states
separately): 1e-4 with fp32 q/k/v/o, 1e-2 with bf16 q/k/v/o. The oracle reads
the same bf16-rounded inputs, upcast exactly.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from linear_attention_sequence_delta_b200 import gdn_prefill, gdn_sync_status
from linear_attention_sequence_delta_b200.inputs import WORKLOADS, make_prefill_inputs
from tests.parity_util import TOL_BF16, TOL_FP32, oracle_prefill_heads, rel_err

pytestmark = pytest.mark.gpu


def _run(P, scale=1.0):
    Pd = P.to("cuda")
    o, Sf = gdn_prefill(Pd.q, Pd.k, Pd.v, Pd.a, Pd.b, Pd.A_log, Pd.dt_bias, Pd.cu_seqlens,
                        Pd.initial_state, scale=scale)
    assert gdn_sync_status() == 0
    return o, Sf


def _full_oracle(P, scale=1.0):
    return oracle.forward(P.q, P.k, P.v, P.a, P.b, P.A_log, P.dt_bias,
                          P.cu_seqlens.cpu().numpy(), P.initial_state, scale=scale)


def _check(P, tol, scale=1.0):
    o, Sf = _run(P, scale)
    o_ref, S_ref = _full_oracle(P, scale)
    eo, es = rel_err(o, o_ref), rel_err(Sf, S_ref)
    assert eo <= tol and es <= tol, (eo, es)
    return eo, es


def test_tiny_fp32_workload():
    """B=1, T=256, 2 QK / 4 V heads, d=64, fp32 I/O: the 1e-4 precision mode."""
    P = make_prefill_inputs(**WORKLOADS["tiny_fp32"], seed=0)
    _check(P, TOL_FP32)


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 127, 200])
def test_ragged_lengths(T, io):
    P = make_prefill_inputs([T], H_qk=2, H_v=4, d_k=128, d_v=128, io_dtype=io, state_std=0.05,
                            seed=T)
    _check(P, TOL_FP32 if io == torch.float32 else TOL_BF16)


@pytest.mark.parametrize("d", [64, 128])
def test_varlen_with_empty_sequences(d):
    P = make_prefill_inputs([70, 0, 1, 64, 129, 0, 5], H_qk=1, H_v=3, d_k=d, d_v=d,
                            io_dtype=torch.float32, state_std=0.1, seed=11)
    _check(P, TOL_FP32)


def test_slow_decay_long_carry():
    """A_log = -4 (alpha near 0.98 per token) keeps state alive across many chunks."""
    P = make_prefill_inputs([777], H_qk=2, H_v=4, d_k=128, d_v=128, io_dtype=torch.float32,
                            seed=3)
    P.A_log.fill_(-4.0)
    _check(P, TOL_FP32)
    Pb = make_prefill_inputs([777], H_qk=2, H_v=4, d_k=128, d_v=128, seed=3)
    Pb.A_log.fill_(-4.0)
    _check(Pb, TOL_BF16)


def test_pages_init_distribution_and_strong_writes():
    """A_log = log U(0, 16) as in the pages' parameter init, beta near 1 (b = 4)."""
    P = make_prefill_inputs([300], H_qk=2, H_v=4, d_k=128, d_v=128, io_dtype=torch.float32,
                            seed=4)
    g = torch.Generator().manual_seed(9)
    P.A_log.copy_(torch.log(torch.rand(4, generator=g) * 16 + 1e-3))
    P.b.fill_(4.0)
    _check(P, TOL_FP32)


def test_extreme_gates():
    """alpha = 1 (a -> -inf), beta = 0 (b -> -inf) and alpha = 0 (A_log = 100) tokens."""
    P = make_prefill_inputs([150], H_qk=1, H_v=3, d_k=64, d_v=64, io_dtype=torch.float32,
                            state_std=0.1, seed=8)
    P.a[10:20, 0] = -1e30
    P.b[30:40, 1] = -1e30
    P.A_log[2] = 100.0
    _check(P, TOL_FP32)


def test_scale_and_final_state_alias():
    P = make_prefill_inputs([100, 37], H_qk=2, H_v=4, d_k=64, d_v=64, io_dtype=torch.float32,
                            state_std=0.1, seed=21)
    Pd = P.to("cuda")
    S = Pd.initial_state.clone()
    o, Sf = gdn_prefill(Pd.q, Pd.k, Pd.v, Pd.a, Pd.b, Pd.A_log, Pd.dt_bias, Pd.cu_seqlens, S,
                        scale=0.125, final_state=S)
    assert Sf.data_ptr() == S.data_ptr()
    o_ref, S_ref = _full_oracle(P, scale=0.125)
    assert rel_err(o, o_ref) <= TOL_FP32 and rel_err(S, S_ref) <= TOL_FP32


def test_split_prefill_resume_equals_single():
    P = make_prefill_inputs([300], H_qk=2, H_v=4, d_k=128, d_v=128, io_dtype=torch.float32,
                            seed=5)
    Pd = P.to("cuda")
    args = lambda s: (Pd.q[s], Pd.k[s], Pd.v[s], Pd.a[s], Pd.b[s], Pd.A_log, Pd.dt_bias)
    cu = lambda n: torch.tensor([0, n], dtype=torch.int32, device="cuda")
    o, Sf = gdn_prefill(*args(slice(0, 300)), cu(300))
    o1, S1 = gdn_prefill(*args(slice(0, 130)), cu(130))
    o2, S2 = gdn_prefill(*args(slice(130, 300)), cu(170), S1)
    torch.cuda.synchronize()
    assert rel_err(torch.cat([o1, o2]), o.cpu().numpy()) <= 1e-5
    assert rel_err(S2, Sf.cpu().numpy()) <= 1e-5


def test_bad_seqlens_reported_on_device():
    P = make_prefill_inputs([64, 64], H_qk=1, H_v=2, d_k=64, d_v=64, io_dtype=torch.float32)
    Pd = P.to("cuda")
    bad = torch.tensor([0, 100, 90], dtype=torch.int32, device="cuda")  # decreasing
    gdn_prefill(Pd.q, Pd.k, Pd.v, Pd.a, Pd.b, Pd.A_log, Pd.dt_bias, bad)
    assert gdn_sync_status() == 6
    assert gdn_sync_status() == 0  # cleared


# ---------------------------------------------------------- full workloads ----

def test_prefill_35b_layer_full():
    """B=1, T=4096, 16 QK / 32 V heads, d=128, bf16: every output against the oracle."""
    P = make_prefill_inputs(**WORKLOADS["prefill_35b"], seed=0)
    _check(P, TOL_BF16)


def test_prefill_397b_long_sampled():
    """B=4, T=16384, 16 QK / 64 V heads: the full launch, sampled (sequence, head) units."""
    P = make_prefill_inputs(**WORKLOADS["prefill_397b_long"], seed=0, device="cuda")
    o, Sf = gdn_prefill(P.q, P.k, P.v, P.a, P.b, P.A_log, P.dt_bias, P.cu_seqlens, None)
    assert gdn_sync_status() == 0
    units = [(0, 0), (1, 17), (3, 63)]
    ref = {}
    for n, h in units:
        ref.update(oracle_prefill_heads(P, [h], seqs=[n]))
    cu = P.cu_seqlens.cpu().tolist()
    for (n, h), (o_ref, S_ref) in ref.items():
        assert rel_err(o[cu[n]:cu[n + 1], h], o_ref) <= TOL_BF16
        assert rel_err(Sf[n, h], S_ref) <= TOL_BF16
    assert torch.isfinite(o.float()).all() and torch.isfinite(Sf).all()


def test_varlen_64_sampled():
    """64 sequences, lengths U[128, 8192], nonzero initial states: sampled units."""
    P = make_prefill_inputs(**WORKLOADS["varlen_64"], seed=0, device="cuda")
    o, Sf = gdn_prefill(P.q, P.k, P.v, P.a, P.b, P.A_log, P.dt_bias, P.cu_seqlens,
                        P.initial_state)
    assert gdn_sync_status() == 0
    cu = P.cu_seqlens.cpu().tolist()
    lens = np.diff(cu)
    seqs = [int(np.argmin(lens)), int(np.argmax(lens)), 31]
    ref = oracle_prefill_heads(P, [0, 13, 31], seqs=seqs)
    for (n, h), (o_ref, S_ref) in ref.items():
        assert rel_err(o[cu[n]:cu[n + 1], h], o_ref) <= TOL_BF16
        assert rel_err(Sf[n, h], S_ref) <= TOL_BF16
    assert torch.isfinite(o.float()).all() and torch.isfinite(Sf).all()


@pytest.fixture
def impl_switch():
    from linear_attention_sequence_delta_b200 import gdn
    prev = gdn.set_prefill_impl(gdn.GDN_IMPL_AUTO)
    yield gdn
    gdn.set_prefill_impl(prev)


IMPLS = {"cuda_core": "GDN_IMPL_CUDA_CORE", "tensor_core": "GDN_IMPL_TENSOR_CORE",
         "tensor_core_split": "GDN_IMPL_TENSOR_CORE_SPLIT",
         "tensor_core_whole_rows": "GDN_IMPL_TENSOR_CORE_WHOLE_ROWS",
         "tensor_core_gram": "GDN_IMPL_TENSOR_CORE_GRAM"}


@pytest.mark.parametrize("impl", list(IMPLS))
@pytest.mark.parametrize("lengths", [[1], [63], [64], [65], [127], [200], [5, 0, 130, 64]])
def test_bf16_every_implementation(impl_switch, impl, lengths):
    g = impl_switch
    g.set_prefill_impl(getattr(g, IMPLS[impl]))
    P = make_prefill_inputs(lengths, H_qk=2, H_v=4, d_k=128, d_v=128, state_std=0.05,
                            seed=sum(lengths) + 7)
    _check(P, TOL_BF16)


@pytest.mark.parametrize("impl", ["GDN_IMPL_TENSOR_CORE", "GDN_IMPL_TENSOR_CORE_GRAM"])
def test_tensor_core_stress_gates(impl_switch, impl):
    """Slow decay, strong writes and extreme gates through the tensor-core path."""
    g = impl_switch
    g.set_prefill_impl(getattr(g, impl))
    P = make_prefill_inputs([500], H_qk=1, H_v=4, d_k=128, d_v=128, state_std=0.1, seed=12)
    P.A_log[0] = -4.0                 # alpha near 0.98: long carry across chunks
    P.b[:, 1] = 4.0                   # beta near 1
    P.a[100:130, 2] = -1e30           # alpha = 1 run
    P.A_log[3] = 100.0                # alpha = 0 every token
    _check(P, TOL_BF16)


def test_tensor_core_rejects_fp32(impl_switch):
    g = impl_switch
    g.set_prefill_impl(g.GDN_IMPL_TENSOR_CORE)
    P = make_prefill_inputs([64], H_qk=1, H_v=1, d_k=128, d_v=128, io_dtype=torch.float32)
    with pytest.raises(g.GDNError):
        _run(P)


def test_kernel_timing_names_and_durations(impl_switch):
    g = impl_switch
    P = make_prefill_inputs([300, 77], H_qk=2, H_v=4, d_k=128, d_v=128, seed=31)
    prev = g.set_kernel_timing(True)
    try:
        for impl, names in ((g.GDN_IMPL_TENSOR_CORE, ["fused_half_rows"]),  # 8 chains
                            (g.GDN_IMPL_TENSOR_CORE_GRAM, ["fused_half_rows_gram"]),
                            (g.GDN_IMPL_TENSOR_CORE_WHOLE_ROWS, ["fused"]),
                            (g.GDN_IMPL_TENSOR_CORE_SPLIT, ["chunk_offsets", "prep", "chain"]),
                            (g.GDN_IMPL_CUDA_CORE, ["gates", "prefill_simt"])):
            g.set_prefill_impl(impl)
            _run(P)
            times = g.last_prefill_kernel_times()
            assert [n for n, _ in times] == names
            assert all(0.0 < ms < 1000.0 for _, ms in times)
    finally:
        g.set_kernel_timing(prev)


@pytest.mark.parametrize("wl", ["prefill_35b", "varlen_64"])
def test_fused_equals_split(impl_switch, wl):
    """The overlapped single launch (half-row chain blocks for the 35B layer's 32 chains,
    whole-row blocks for 64 chains) and the separate launches compute the same thing
    (same arithmetic per element, different scheduling): outputs agree to the last bit."""
    g = impl_switch
    W = dict(WORKLOADS[wl])
    if wl == "varlen_64":
        W["num_seqs"] = 2  # 64 chains: few enough for the overlapped launch
    P = make_prefill_inputs(**W, seed=3, device="cuda")
    fused = "fused_half_rows" if wl == "prefill_35b" else "fused"
    outs = []
    prev = g.set_kernel_timing(True)
    try:
        for impl, kernel in ((g.GDN_IMPL_TENSOR_CORE, fused),
                             (g.GDN_IMPL_TENSOR_CORE_WHOLE_ROWS, "fused"),
                             (g.GDN_IMPL_TENSOR_CORE_SPLIT, "chain")):
            g.set_prefill_impl(impl)
            o, Sf = gdn_prefill(P.q, P.k, P.v, P.a, P.b, P.A_log, P.dt_bias, P.cu_seqlens,
                                P.initial_state)
            assert gdn_sync_status() == 0
            assert kernel in [n for n, _ in g.last_prefill_kernel_times()]
            outs.append((o, Sf))
    finally:
        g.set_kernel_timing(prev)
    for o_, S_ in outs[1:]:
        assert torch.equal(outs[0][0], o_) and torch.equal(outs[0][1], S_)


@pytest.mark.parametrize("lengths,H_qk,H_v", [([4096], 4, 8), ([1000, 300, 64, 2000, 1], 2, 4)])
def test_gram_schedule(impl_switch, lengths, H_qk, H_v):
    """The cross-chunk Gram-matrix schedule (half-row blocks; S_c K_c^T built from the
    previous chunk's bf16 state and the key Gram matrix) against the oracle, every output,
    and against the default schedule: the same mathematics with another bf16 rounding."""
    g = impl_switch
    P = make_prefill_inputs(lengths, H_qk=H_qk, H_v=H_v, d_k=128, d_v=128, state_std=0.05,
                            seed=len(lengths) + 40)
    prev = g.set_kernel_timing(True)
    try:
        g.set_prefill_impl(g.GDN_IMPL_TENSOR_CORE_GRAM)
        o, Sf = _run(P)
        assert [n for n, _ in g.last_prefill_kernel_times()] == ["fused_half_rows_gram"]
        g.set_prefill_impl(g.GDN_IMPL_TENSOR_CORE)
        o_d, S_d = _run(P)
    finally:
        g.set_kernel_timing(prev)
    o_ref, S_ref = _full_oracle(P)
    assert rel_err(o, o_ref) <= TOL_BF16 and rel_err(Sf, S_ref) <= TOL_BF16
    # both schedules sit well inside the tolerance and close to each other
    assert rel_err(o, o_d.float().cpu().numpy()) <= TOL_BF16 / 2
    assert rel_err(Sf, S_d.cpu().numpy()) <= TOL_BF16 / 2


def test_gram_schedule_35b_layer_full(impl_switch):
    g = impl_switch
    g.set_prefill_impl(g.GDN_IMPL_TENSOR_CORE_GRAM)
    P = make_prefill_inputs(**WORKLOADS["prefill_35b"], seed=0)
    _check(P, TOL_BF16)


def test_many_chains_use_separate_launches(impl_switch):
    """With more (sequence, V head) chains than half the SMs the default path runs the
    preparation and the chains as separate launches."""
    g = impl_switch
    g.set_prefill_impl(g.GDN_IMPL_AUTO)
    P = make_prefill_inputs([100] * 8, H_qk=16, H_v=32, d_k=128, d_v=128, seed=4)
    prev = g.set_kernel_timing(True)
    try:
        _check(P, TOL_BF16)
        assert [n for n, _ in g.last_prefill_kernel_times()] == ["chunk_offsets", "prep", "chain"]
    finally:
        g.set_kernel_timing(prev)
