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
from linear_attention_sequence_delta_b200 import gdn, gdn_prefill, gdn_sync_status
from linear_attention_sequence_delta_b200.inputs import WORKLOADS, make_prefill_inputs
from tests.parity_util import TOL_BF16, TOL_FP32, rel_err

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


def _check_per_sequence(P, o, Sf):
    """Every output and final state against the oracle, one oracle call per sequence
    (all V heads of it at once, OpenMP over the heads): exact, since (sequence, head)
    units are independent, and the host memory stays bounded."""
    cu = P.cu_seqlens.cpu().tolist()
    worst_o = worst_s = 0.0
    for n in range(len(cu) - 1):
        s0, s1 = cu[n], cu[n + 1]
        S0 = None if P.initial_state is None else P.initial_state[n:n + 1].cpu()
        o_ref, S_ref = oracle.forward(P.q[s0:s1].cpu(), P.k[s0:s1].cpu(), P.v[s0:s1].cpu(),
                                      P.a[s0:s1].cpu(), P.b[s0:s1].cpu(), P.A_log.cpu(),
                                      P.dt_bias.cpu(), [0, s1 - s0], S0)
        eo, es = rel_err(o[s0:s1], o_ref), rel_err(Sf[n:n + 1], S_ref)
        assert eo <= TOL_BF16 and es <= TOL_BF16, (n, eo, es)
        worst_o, worst_s = max(worst_o, eo), max(worst_s, es)
    return worst_o, worst_s


def test_prefill_397b_long_full():
    """B=4, T=16384, 16 QK / 64 V heads, d=128, bf16: every output and final state of
    all 256 (sequence, head) units against the oracle."""
    P = make_prefill_inputs(**WORKLOADS["prefill_397b_long"], seed=0, device="cuda")
    o, Sf = gdn_prefill(P.q, P.k, P.v, P.a, P.b, P.A_log, P.dt_bias, P.cu_seqlens, None)
    assert gdn_sync_status() == 0
    _check_per_sequence(P, o, Sf)


def test_varlen_64_full():
    """64 sequences, lengths U[128, 8192], nonzero initial states: all 2,048 units."""
    P = make_prefill_inputs(**WORKLOADS["varlen_64"], seed=0, device="cuda")
    o, Sf = gdn_prefill(P.q, P.k, P.v, P.a, P.b, P.A_log, P.dt_bias, P.cu_seqlens,
                        P.initial_state)
    assert gdn_sync_status() == 0
    _check_per_sequence(P, o, Sf)


IMPLS = {"cuda_core": gdn.GDN_IMPL_CUDA_CORE, "tensor_core": gdn.GDN_IMPL_TENSOR_CORE,
         "tensor_core_split": gdn.GDN_IMPL_TENSOR_CORE_SPLIT,
         "tensor_core_whole_rows": gdn.GDN_IMPL_TENSOR_CORE_WHOLE_ROWS}


def _check_impl(P, impl, tol=TOL_BF16, timer=None):
    Pd = P.to("cuda")
    o, Sf = gdn_prefill(Pd.q, Pd.k, Pd.v, Pd.a, Pd.b, Pd.A_log, Pd.dt_bias, Pd.cu_seqlens,
                        Pd.initial_state, impl=impl, timer=timer)
    assert gdn_sync_status() == 0
    o_ref, S_ref = _full_oracle(P)
    eo, es = rel_err(o, o_ref), rel_err(Sf, S_ref)
    assert eo <= tol and es <= tol, (eo, es)
    return o, Sf


@pytest.mark.parametrize("impl", list(IMPLS))
@pytest.mark.parametrize("lengths", [[1], [63], [64], [65], [127], [200], [5, 0, 130, 64]])
def test_bf16_every_implementation(impl, lengths):
    P = make_prefill_inputs(lengths, H_qk=2, H_v=4, d_k=128, d_v=128, state_std=0.05,
                            seed=sum(lengths) + 7)
    _check_impl(P, IMPLS[impl])


@pytest.mark.parametrize("impl", ["tensor_core", "tensor_core_split"])
def test_tensor_core_stress_gates(impl):
    """Slow decay, strong writes and extreme gates through the tensor-core path."""
    P = make_prefill_inputs([500], H_qk=1, H_v=4, d_k=128, d_v=128, state_std=0.1, seed=12)
    P.A_log[0] = -4.0                 # alpha near 0.98: long carry across chunks
    P.b[:, 1] = 4.0                   # beta near 1
    P.a[100:130, 2] = -1e30           # alpha = 1 run
    P.A_log[3] = 100.0                # alpha = 0 every token
    _check_impl(P, IMPLS[impl])


def test_tensor_core_rejects_fp32():
    P = make_prefill_inputs([64], H_qk=1, H_v=1, d_k=128, d_v=128, io_dtype=torch.float32)
    with pytest.raises(gdn.GDNError):
        _check_impl(P, gdn.GDN_IMPL_TENSOR_CORE)


def test_kernel_timing_names_and_durations():
    P = make_prefill_inputs([300, 77], H_qk=2, H_v=4, d_k=128, d_v=128, seed=31)
    timer = gdn.Timer()
    for impl, names in ((gdn.GDN_IMPL_TENSOR_CORE, ["fused_half_rows"]),  # 8 chains
                        (gdn.GDN_IMPL_TENSOR_CORE_WHOLE_ROWS, ["fused"]),
                        (gdn.GDN_IMPL_TENSOR_CORE_SPLIT, ["chunk_offsets", "prep", "chain"]),
                        (gdn.GDN_IMPL_CUDA_CORE, ["gates", "prefill_simt"])):
        _check_impl(P, impl, timer=timer)
        times = timer.times()
        assert [n for n, _ in times] == names
        assert all(0.0 < ms < 1000.0 for _, ms in times)
    # a call without the timer leaves its record alone
    _check_impl(P, gdn.GDN_IMPL_TENSOR_CORE_SPLIT)
    assert [n for n, _ in timer.times()] == ["gates", "prefill_simt"]
    timer.close()


def test_timer_left_open_at_exit():
    """A timer still alive when the interpreter exits is released by its finaliser
    without an error (module globals may already be gone by then)."""
    import os
    import subprocess
    import sys
    code = ("import torch\n"
            "from linear_attention_sequence_delta_b200 import gdn\n"
            "torch.zeros(1, device='cuda')\n"
            "t = gdn.Timer()\n")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                       timeout=300, cwd=root)
    assert r.returncode == 0, r.stderr
    assert "Exception ignored" not in r.stderr and "Error" not in r.stderr, r.stderr


@pytest.mark.parametrize("wl", ["prefill_35b", "varlen_64"])
def test_fused_equals_split(wl):
    """The overlapped single launch (half-row chain blocks for the 35B layer's 32 chains,
    whole-row blocks for 64 chains) and the separate launches compute the same thing
    (same arithmetic per element, different scheduling): outputs agree to the last bit."""
    W = dict(WORKLOADS[wl])
    if wl == "varlen_64":
        W["num_seqs"] = 2  # 64 chains: few enough for the overlapped launch
    P = make_prefill_inputs(**W, seed=3, device="cuda")
    fused = "fused_half_rows" if wl == "prefill_35b" else "fused"
    outs = []
    timer = gdn.Timer()
    for impl, kernel in ((gdn.GDN_IMPL_TENSOR_CORE, fused),
                         (gdn.GDN_IMPL_TENSOR_CORE_WHOLE_ROWS, "fused"),
                         (gdn.GDN_IMPL_TENSOR_CORE_SPLIT, "chain")):
        o, Sf = gdn_prefill(P.q, P.k, P.v, P.a, P.b, P.A_log, P.dt_bias, P.cu_seqlens,
                            P.initial_state, impl=impl, timer=timer)
        assert gdn_sync_status() == 0
        assert kernel in [n for n, _ in timer.times()]
        outs.append((o, Sf))
    for o_, S_ in outs[1:]:
        assert torch.equal(outs[0][0], o_) and torch.equal(outs[0][1], S_)


def test_many_chains_use_separate_launches():
    """With more (sequence, V head) chains than half the SMs the default path runs the
    preparation and the chains as separate launches."""
    P = make_prefill_inputs([100] * 8, H_qk=16, H_v=32, d_k=128, d_v=128, seed=4)
    timer = gdn.Timer()
    _check_impl(P, gdn.GDN_IMPL_AUTO, timer=timer)
    assert [n for n, _ in timer.times()] == ["chunk_offsets", "prep", "chain"]


def test_chain_order_longest_first():
    """The separate launches run the chains of the sequences with the most chunks first:
    the order the offsets kernel leaves in the workspace (after the N + 1 chunk offsets)
    is the sequences by chunk count, most first, ties by index; the results match the
    oracle whatever the order."""
    lens = [100, 700, 0, 64, 65, 700, 1, 300, 128, 129, 5, 640]
    P = make_prefill_inputs(lens, H_qk=4, H_v=8, d_k=128, d_v=128, state_std=0.05, seed=61)
    Pd = P.to("cuda")
    N, T = len(lens), sum(lens)
    work = torch.zeros(gdn.workspace_size(N, T, 4, 8, 128, 128), dtype=torch.uint8,
                       device="cuda")
    o, Sf = gdn_prefill(Pd.q, Pd.k, Pd.v, Pd.a, Pd.b, Pd.A_log, Pd.dt_bias, Pd.cu_seqlens,
                        Pd.initial_state, workspace=work, impl=gdn.GDN_IMPL_TENSOR_CORE_SPLIT)
    assert gdn_sync_status() == 0
    words = work[: (2 * N + 1) * 4].view(torch.int32).cpu().tolist()
    chunks = [(n_ + 63) // 64 for n_ in lens]
    assert words[:N + 1] == [sum(chunks[:i]) for i in range(N + 1)]
    assert words[N + 1:] == sorted(range(N), key=lambda i: (-chunks[i], i))
    o_ref, S_ref = _full_oracle(P)
    assert rel_err(o, o_ref) <= TOL_BF16 and rel_err(Sf, S_ref) <= TOL_BF16


# ------------------------------------------------ workspace contents, failures ----

def _ws_fill(work, pattern):
    """Fill a workspace with contents a caching allocator could hand back."""
    w64 = work[: work.numel() // 8 * 8].view(torch.int64)
    if pattern == "small_ints":      # every small integer, in order
        w64.copy_(torch.arange(w64.numel(), device=work.device, dtype=torch.int64))
    elif pattern == "small_ints_rev":
        w64.copy_(torch.arange(w64.numel(), 0, -1, device=work.device, dtype=torch.int64))
    elif pattern == "ones":
        w64.fill_(1)
    elif pattern == "all_bits":
        work.fill_(0xFF)
    elif pattern == "top_bit":       # the form this library's call numbers take
        w64.fill_(-(1 << 63))


@pytest.mark.parametrize("pattern", ["small_ints", "small_ints_rev", "ones", "all_bits",
                                     "top_bit"])
@pytest.mark.parametrize("lengths,H_v,impl", [([700, 333], 4, gdn.GDN_IMPL_TENSOR_CORE),
                                              ([700, 333], 4, gdn.GDN_IMPL_TENSOR_CORE_WHOLE_ROWS),
                                              ([1000] * 20, 4, gdn.GDN_IMPL_TENSOR_CORE_SPLIT)])
def test_workspace_contents_do_not_matter(pattern, lengths, H_v, impl):
    """A record counts as published only when its flag equals this call's number. A
    workspace that already holds integers (every small value, as indices or counts left
    by other work would), all-ones bytes, or words with only the top bit set, must give
    the same results as a fresh one, compared with the oracle on every output."""
    P = make_prefill_inputs(lengths, H_qk=2, H_v=H_v, d_k=128, d_v=128, state_std=0.05,
                            seed=len(lengths) + 50)
    Pd = P.to("cuda")
    T, N = P.q.shape[0], P.num_seqs
    work = torch.empty(gdn.workspace_size(N, T, 2, H_v, 128, 128), dtype=torch.uint8,
                       device="cuda")
    o_ref, S_ref = _full_oracle(P)
    for _ in range(2):  # refilled before each of two calls in a row
        _ws_fill(work, pattern)
        o, Sf = gdn_prefill(Pd.q, Pd.k, Pd.v, Pd.a, Pd.b, Pd.A_log, Pd.dt_bias, Pd.cu_seqlens,
                            Pd.initial_state, workspace=work, impl=impl)
        assert gdn_sync_status() == 0
        assert rel_err(o, o_ref) <= TOL_BF16 and rel_err(Sf, S_ref) <= TOL_BF16


@pytest.mark.parametrize("lengths,H_v", [([300, 77], 4),      # half-row chain blocks
                                         ([200] * 12, 4)])    # whole-row chain blocks
def test_bounded_wait_runs_out_and_context_survives(lengths, H_v):
    """Fault injection on the host side: the overlapped launch's preparation publishes
    no record, so every chain's bounded wait (here about 10^5 cycles) runs out. The
    call must end by itself with GDN_ERR_TIMEOUT in the status word (nothing traps or
    hangs: each role leaves its loops, drains its copies and frees its tensor memory),
    and the next ordinary call on the same context must match the oracle."""
    P = make_prefill_inputs(lengths, H_qk=2, H_v=H_v, d_k=128, d_v=128, state_std=0.05,
                            seed=len(lengths) + 60)
    Pd = P.to("cuda")
    timer = gdn.Timer()
    for _ in range(2):
        gdn_prefill(Pd.q, Pd.k, Pd.v, Pd.a, Pd.b, Pd.A_log, Pd.dt_bias, Pd.cu_seqlens,
                    Pd.initial_state, fault=gdn.GDN_FAULT_WITHHOLD_RECORDS,
                    wait_limit_cycles=100_000, timer=timer)
        assert gdn_sync_status() == 5  # GDN_ERR_TIMEOUT
        assert gdn_sync_status() == 0  # read and cleared
        (name, ms), = timer.times()
        assert name.startswith("fused") and ms < 100.0  # the short limit, not the default
    o, Sf = _check_impl(P, gdn.GDN_IMPL_AUTO)


def _guarded(shape, dtype, guard=4096):
    """A tensor of `shape` inside a larger buffer whose guard regions (`guard` bytes on
    each side) hold a known pattern."""
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    buf = torch.empty(n + 2 * guard, dtype=torch.uint8, device="cuda")
    buf.fill_(0xA5)
    t = buf[guard:guard + n].view(dtype).view(shape)
    return buf, t


def _guards_intact(buf, guard=4096):
    return bool((buf[:guard] == 0xA5).all() and (buf[-guard:] == 0xA5).all())


@pytest.mark.parametrize("impl,lengths,io", [
    (gdn.GDN_IMPL_TENSOR_CORE, [70, 0, 1, 130], torch.bfloat16),
    (gdn.GDN_IMPL_TENSOR_CORE_WHOLE_ROWS, [70, 0, 1, 130], torch.bfloat16),
    (gdn.GDN_IMPL_TENSOR_CORE_SPLIT, [70, 0, 1, 130], torch.bfloat16),
    (gdn.GDN_IMPL_CUDA_CORE, [70, 0, 1, 130], torch.float32)])
def test_outputs_stay_inside_their_buffers(impl, lengths, io):
    """Guard regions around o and the final states (a stand-in for a memory checker):
    ragged tails, empty and one-token sequences write nothing outside the outputs."""
    P = make_prefill_inputs(lengths, H_qk=2, H_v=4, d_k=128, d_v=128, io_dtype=io,
                            state_std=0.05, seed=70)
    Pd = P.to("cuda")
    T, N = P.q.shape[0], P.num_seqs
    ob, o = _guarded((T, 4, 128), io)
    sb, Sf = _guarded((N, 4, 128, 128), torch.float32)
    gdn_prefill(Pd.q, Pd.k, Pd.v, Pd.a, Pd.b, Pd.A_log, Pd.dt_bias, Pd.cu_seqlens,
                Pd.initial_state, out=o, final_state=Sf, impl=impl)
    assert gdn_sync_status() == 0
    assert _guards_intact(ob) and _guards_intact(sb)
    o_ref, S_ref = _full_oracle(P)
    tol = TOL_BF16 if io == torch.bfloat16 else TOL_FP32
    assert rel_err(o, o_ref) <= tol and rel_err(Sf, S_ref) <= tol
