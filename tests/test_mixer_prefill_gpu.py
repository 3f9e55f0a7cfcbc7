"""gdn_mixer_prefill (the causal conv1d + SiLU fused into the prefill's preparation, the
gated RMSNorm fused into the chain's output) against the fp64 oracle's steps composed:
oracle.conv1d_silu -> (rounded to the I/O type, split into q | k | v) -> oracle.forward ->
oracle.rmsnorm_gated ("Qwen3.5-MoE-35B-A3B architecture teardown", 3.3 phases 2-4;
"Qwen3.5 observation notes", "Qwen3_5MoeGatedDeltaNet").

Tolerance: max|gpu - oracle| / max|oracle| <= 1e-2 (bf16 I/O) or 1e-4 (fp32 I/O), on y
and on the final states separately; the conv cache holds copies of inputs and is
compared bit for bit.
"""
import numpy as np
import pytest
import torch

from linear_attention_sequence_delta_b200 import (gdn, gdn_conv1d_silu, gdn_mixer_prefill,
                                                  gdn_prefill, gdn_rmsnorm_gated,
                                                  gdn_sync_status)
from linear_attention_sequence_delta_b200.inputs import make_mixer_prefill_inputs
from tests.parity_util import TOL_BF16, TOL_FP32, oracle_mixer, rel_err

pytestmark = pytest.mark.gpu


def _run(P, impl=gdn.GDN_IMPL_AUTO, in_place=False, cache=True, timer=None, eps=1e-6):
    Pd = P.to("cuda")
    cin = Pd.conv_state.clone() if cache else None
    cout = cin if (in_place and cache) else torch.empty_like(Pd.conv_state)
    y, Sf = gdn_mixer_prefill(Pd.x, Pd.conv_weight, Pd.conv_bias, Pd.cu_seqlens, Pd.a, Pd.b,
                              Pd.A_log, Pd.dt_bias, Pd.z, Pd.norm_weight, H_qk=P.H_qk,
                              conv_state_in=cin, conv_state_out=cout,
                              initial_state=Pd.initial_state, eps=eps, impl=impl, timer=timer)
    assert gdn_sync_status() == 0
    return y, Sf, cout


def _check(P, tol, **kw):
    y, Sf, cout = _run(P, **kw)
    Pr = P if kw.get("cache", True) else _no_cache(P)
    y_ref, S_ref, c_ref = oracle_mixer(Pr)
    ey, es = rel_err(y, y_ref), rel_err(Sf, S_ref)
    assert ey <= tol and es <= tol, (ey, es)
    assert np.array_equal(cout.float().cpu().numpy(), c_ref), "conv cache"
    return y, Sf, cout


def _no_cache(P):
    import dataclasses
    return dataclasses.replace(P, conv_state=torch.zeros_like(P.conv_state))


@pytest.mark.parametrize("impl,kernels", [
    (gdn.GDN_IMPL_AUTO, ["conv1d_silu", "fused_half_rows", "rmsnorm_gated"]),
    (gdn.GDN_IMPL_TENSOR_CORE, ["fused"])])
def test_mixer_35b_layer(impl, kernels):
    """The 35B-A3B layer (T=4096, 16 QK / 32 V heads, d=128, K=4), conv cache in and
    out, initial states in: by default the convolution, the prefill (overlapped, half-row
    chain blocks) and the norm; with the fused schedule one overlapped launch."""
    P = make_mixer_prefill_inputs([4096], H_qk=16, H_v=32, d=128, state_std=0.02, seed=1)
    timer = gdn.Timer()
    _check(P, TOL_BF16, impl=impl, timer=timer)
    assert [n for n, _ in timer.times()] == kernels


@pytest.mark.parametrize("K", [2, 3, 4])
@pytest.mark.parametrize("impl", [gdn.GDN_IMPL_AUTO, gdn.GDN_IMPL_TENSOR_CORE,
                                  gdn.GDN_IMPL_TENSOR_CORE_SPLIT])
def test_mixer_ragged_and_short(K, impl):
    """Empty sequences, sequences shorter than the cache, one token, a whole chunk, a
    ragged tail; overlapped and separate launches."""
    P = make_mixer_prefill_inputs([70, 0, 1, 2, 64, 129, 300], H_qk=2, H_v=4, d=128,
                                  kernel_size=K, state_std=0.05, seed=10 + K)
    _check(P, TOL_BF16, impl=impl)


@pytest.mark.parametrize("impl", [gdn.GDN_IMPL_AUTO, gdn.GDN_IMPL_TENSOR_CORE,
                                  gdn.GDN_IMPL_TENSOR_CORE_SPLIT])
def test_mixer_cache_in_place_and_absent(impl):
    P = make_mixer_prefill_inputs([130, 1, 0, 65], H_qk=2, H_v=8, d=128, state_std=0.05,
                                  seed=21)
    _check(P, TOL_BF16, impl=impl, in_place=True)
    P2 = make_mixer_prefill_inputs([130, 1, 0, 65], H_qk=2, H_v=8, d=128, seed=22)
    _check(P2, TOL_BF16, impl=impl, cache=False)


@pytest.mark.parametrize("impl,kernels", [
    (gdn.GDN_IMPL_AUTO, ["conv1d_silu", "chunk_offsets", "prep", "chain", "rmsnorm_gated"]),
    (gdn.GDN_IMPL_TENSOR_CORE, ["conv1d_silu", "chunk_offsets", "prep", "chain"])])
def test_mixer_many_chains_separate_launches(impl, kernels):
    """More chains than half the SMs: the convolution as its own streaming kernel, then
    preparation and chains as separate launches, and the norm as its own kernel (by
    default) or in the chains' output (fused schedule)."""
    P = make_mixer_prefill_inputs([300] * 6, H_qk=16, H_v=32, d=128, state_std=0.02, seed=5)
    timer = gdn.Timer()
    _check(P, TOL_BF16, impl=impl, timer=timer)
    assert [n for n, _ in timer.times()] == kernels


@pytest.mark.parametrize("lengths,d", [([100, 0, 37], 64), ([70, 3], 128)])
def test_mixer_fp32_runs_the_steps_in_turn(lengths, d):
    P = make_mixer_prefill_inputs(lengths, H_qk=2, H_v=4, d=d, io_dtype=torch.float32,
                                  state_std=0.05, seed=31)
    timer = gdn.Timer()
    _check(P, TOL_FP32, timer=timer)
    assert [n for n, _ in timer.times()] == ["conv1d_silu", "gates", "prefill_simt",
                                             "rmsnorm_gated"]


@pytest.mark.parametrize("impl", [gdn.GDN_IMPL_AUTO, gdn.GDN_IMPL_TENSOR_CORE])
def test_mixer_equals_the_three_calls(impl):
    """The call against gdn_conv1d_silu -> gdn_prefill -> gdn_rmsnorm_gated on the GPU:
    the default schedule runs those kernels (the prefill reading the post-conv buffer with
    a token stride), so everything agrees to the last bit; in the fused schedule the
    convolution has the same arithmetic (same q, k, v bits), so the final states and the
    conv cache agree to the last bit and y differs only by the norm's order of summation
    (within one bf16 rounding)."""
    P = make_mixer_prefill_inputs([700, 64, 1, 333], H_qk=4, H_v=8, d=128, state_std=0.05,
                                  seed=41)
    y, Sf, cout = _run(P, impl=impl)
    Pd = P.to("cuda")
    yc, c2 = gdn_conv1d_silu(Pd.x, Pd.conv_weight, Pd.conv_bias, Pd.cu_seqlens, Pd.conv_state)
    T, C = Pd.x.shape
    H_qk, H_v, d = P.H_qk, Pd.z.shape[1], Pd.z.shape[2]
    q = yc[:, :H_qk * d].reshape(T, H_qk, d).contiguous()
    k = yc[:, H_qk * d:2 * H_qk * d].reshape(T, H_qk, d).contiguous()
    v = yc[:, 2 * H_qk * d:].reshape(T, H_v, d).contiguous()
    o, S2 = gdn_prefill(q, k, v, Pd.a, Pd.b, Pd.A_log, Pd.dt_bias, Pd.cu_seqlens,
                        Pd.initial_state)
    y2 = gdn_rmsnorm_gated(o, Pd.z, Pd.norm_weight, 1e-6)
    assert gdn_sync_status() == 0
    assert torch.equal(Sf, S2)
    assert torch.equal(cout, c2)
    if impl == gdn.GDN_IMPL_AUTO:
        assert torch.equal(y, y2)
    dy = (y.float() - y2.float()).abs()
    assert bool((dy <= 2.0 ** -7 * y2.float().abs() + 1e-3).all()), float(dy.max())


@pytest.mark.parametrize("impl", [gdn.GDN_IMPL_AUTO, gdn.GDN_IMPL_TENSOR_CORE,
                                  gdn.GDN_IMPL_TENSOR_CORE_SPLIT])
def test_mixer_writes_nothing_outside_its_outputs(impl):
    """Guard regions around y and the conv cache (a stand-in for a memory checker)."""
    P = make_mixer_prefill_inputs([70, 0, 1, 130], H_qk=2, H_v=4, d=128, state_std=0.05,
                                  seed=51)
    Pd = P.to("cuda")
    G = 4096

    def guarded(t):
        n = t.numel() * t.element_size()
        buf = torch.full((n + 2 * G,), 0xA5, dtype=torch.uint8, device="cuda")
        return buf, buf[G:G + n].view(t.dtype).view(t.shape)

    yb, y = guarded(Pd.z)
    cb, cout = guarded(Pd.conv_state)
    gdn_mixer_prefill(Pd.x, Pd.conv_weight, Pd.conv_bias, Pd.cu_seqlens, Pd.a, Pd.b, Pd.A_log,
                      Pd.dt_bias, Pd.z, Pd.norm_weight, H_qk=P.H_qk, conv_state_in=Pd.conv_state,
                      conv_state_out=cout, initial_state=Pd.initial_state, out=y, impl=impl)
    assert gdn_sync_status() == 0
    for b in (yb, cb):
        assert bool((b[:G] == 0xA5).all() and (b[-G:] == 0xA5).all())
    y_ref, S_ref, c_ref = oracle_mixer(P)
    assert rel_err(y, y_ref) <= TOL_BF16
