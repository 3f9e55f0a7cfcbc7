"""The steps around the delta rule on the GPU, against the fp64 oracle: the causal
depthwise conv1d + SiLU with its per-sequence cache ("Qwen3.5-MoE-35B-A3B architecture
teardown", 3.3 phase 2, 3.4) and the gated RMSNorm (3.3 phase 4).

Tolerances. Both kernels compute in fp32 from inputs that the oracle reads exactly, so
the only error of note is the final rounding to the I/O type: per element
|gpu - oracle| <= 2^-8 |oracle| + 1e-5 for bf16 output (half an ulp is 2^-9), and
<= 1e-5 |oracle| + 1e-6 for fp32 output; on top, the aggregate bar
max|gpu - oracle| / max|oracle| <= 1e-2 (bf16) and 1e-4 (fp32). The conv cache holds
copies of inputs and is compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_sequence_delta_b200 import (GDNError, gdn_conv1d_silu,
                                                  gdn_conv1d_silu_decode, gdn_rmsnorm_gated,
                                                  gdn_sync_status)
from linear_attention_sequence_delta_b200.inputs import make_mixer_inputs
from tests.parity_util import TOL_BF16, TOL_FP32, rel_err

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _close(gpu, ref, dtype):
    g = _np(gpu)
    ref = np.asarray(ref, dtype=np.float64)
    if dtype == torch.bfloat16:
        rel, ab, tol = 2.0 ** -8, 1e-5, TOL_BF16
    else:
        rel, ab, tol = 1e-5, 1e-6, TOL_FP32
    bad = np.abs(g - ref) > rel * np.abs(ref) + ab
    assert not bad.any(), (int(bad.sum()), np.argwhere(bad)[:5], g[bad][:5], ref[bad][:5])
    assert rel_err(gpu, ref) <= tol


def _conv(M, K=4, bias=False, cache=True, want_state=True, cu=None):
    Md = M.to("cuda")
    w = Md.conv_weight[:, :K].contiguous()
    st = Md.conv_state[:, :K - 1].contiguous() if cache else None
    y, so = gdn_conv1d_silu(Md.x, w, Md.conv_bias if bias else None,
                            Md.cu_seqlens if cu is None else cu, st, want_state=want_state)
    assert gdn_sync_status() == 0
    return y, so


def _conv_ref(M, K=4, bias=False, cache=True, want_state=True):
    return oracle.conv1d_silu(M.x, M.conv_weight[:, :K], M.conv_bias if bias else None,
                              M.cu_seqlens.numpy(),
                              M.conv_state[:, :K - 1] if cache else None, want_state=want_state)


# ------------------------------------------------------------------ conv1d + SiLU --

def test_conv_35b_shape_bf16():
    """One 4096-token sequence over the 35B-A3B conv_dim (2*16*128 + 32*128 = 8192)."""
    M = make_mixer_inputs(num_seqs=1, seq_len=4096, seed=1)
    y, so = _conv(M, cache=False)
    y_ref, so_ref = _conv_ref(M, cache=False)
    _close(y, y_ref, torch.bfloat16)
    np.testing.assert_array_equal(_np(so), so_ref)


@pytest.mark.parametrize("K", [2, 3, 4])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_conv_varlen_cache_bias(K, dtype):
    """Packed sequences of every length class: empty, shorter than the cache, inside one
    token tile, crossing tiles, with a ragged tail; a bias; a cache in and out."""
    lens = [5, 0, 1, 2, 9, 40, 0, 33, 16, 17, 3, 100]
    M = make_mixer_inputs(lens, H_qk=2, H_v=4, d_k=64, d_v=64, io_dtype=dtype, seed=2)
    y, so = _conv(M, K=K, bias=True)
    y_ref, so_ref = _conv_ref(M, K=K, bias=True)
    _close(y, y_ref, dtype)
    np.testing.assert_array_equal(_np(so), so_ref)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_conv_narrow_channels(dtype):
    """conv_dim = 24 (three 8-channel vectors): one warp spans several token tiles and the
    grid's last block is partly empty (bf16 and fp32)."""
    lens = [70, 0, 2, 33]
    M = make_mixer_inputs(lens, H_qk=1, H_v=1, d_k=8, d_v=8, io_dtype=dtype, seed=14)
    assert M.x.shape[1] == 24
    y, so = _conv(M, bias=True)
    y_ref, so_ref = _conv_ref(M, bias=True)
    _close(y, y_ref, dtype)
    np.testing.assert_array_equal(_np(so), so_ref)


def test_conv_no_state_out_and_zero_cache():
    M = make_mixer_inputs([7, 300, 1], H_qk=2, H_v=4, d_k=64, d_v=64, seed=3)
    y, so = _conv(M, cache=False, want_state=False)
    assert so is None
    y_ref, _ = _conv_ref(M, cache=False, want_state=False)
    _close(y, y_ref, torch.bfloat16)


def test_conv_chaining_is_bit_exact():
    """prefill(T1) then prefill(T2) from its cache gives the one-pass outputs and cache
    bit for bit (every output is the same fp32 expression of the same inputs)."""
    M = make_mixer_inputs(num_seqs=1, seq_len=200, H_qk=2, H_v=4, d_k=64, d_v=64, seed=4)
    Md = M.to("cuda")
    w = Md.conv_weight
    y, so = gdn_conv1d_silu(Md.x, w, None, Md.cu_seqlens, Md.conv_state)
    for split in (1, 3, 16, 77):
        cu1 = torch.tensor([0, split], dtype=torch.int32, device="cuda")
        cu2 = torch.tensor([0, 200 - split], dtype=torch.int32, device="cuda")
        y1, s1 = gdn_conv1d_silu(Md.x[:split].contiguous(), w, None, cu1, Md.conv_state)
        y2, s2 = gdn_conv1d_silu(Md.x[split:].contiguous(), w, None, cu2, s1)
        assert torch.equal(torch.cat([y1, y2]), y)
        assert torch.equal(s2, so)
    assert gdn_sync_status() == 0


def test_conv_state_in_place():
    M = make_mixer_inputs([3, 1, 0, 50], H_qk=2, H_v=4, d_k=64, d_v=64, seed=5)
    Md = M.to("cuda")
    st = Md.conv_state.clone()
    y, so = gdn_conv1d_silu(Md.x, Md.conv_weight, Md.conv_bias, Md.cu_seqlens, st,
                            conv_state_out=st)
    assert so.data_ptr() == st.data_ptr()
    assert gdn_sync_status() == 0
    y_ref, so_ref = _conv_ref(M, bias=True)
    _close(y, y_ref, torch.bfloat16)
    np.testing.assert_array_equal(_np(st), so_ref)


def test_conv_decode_matches_prefill_and_oracle():
    """Token-by-token decode from a prefill's cache equals the one-pass prefill, bit for
    bit, and the oracle within tolerance; the cache slides in place."""
    lens = [37, 5, 64]
    steps = 6
    M = make_mixer_inputs([L + steps for L in lens], H_qk=2, H_v=4, d_k=64, d_v=64, seed=6)
    Md = M.to("cuda")
    cu = M.cu_seqlens.tolist()
    y_all, _ = gdn_conv1d_silu(Md.x, Md.conv_weight, Md.conv_bias, Md.cu_seqlens, Md.conv_state)
    # prefill of the first lens[n] tokens of each sequence
    idx = torch.cat([torch.arange(cu[n], cu[n] + L) for n, L in enumerate(lens)])
    cu_p = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    _, cache = gdn_conv1d_silu(Md.x[idx.cuda()].contiguous(), Md.conv_weight, Md.conv_bias, cu_p,
                               Md.conv_state)
    for s in range(steps):
        tok = torch.tensor([cu[n] + L + s for n, L in enumerate(lens)], device="cuda")
        yd = gdn_conv1d_silu_decode(Md.x[tok].contiguous(), Md.conv_weight, Md.conv_bias, cache)
        assert torch.equal(yd, y_all[tok])
    assert gdn_sync_status() == 0
    y_ref, so_ref = _conv_ref(M, bias=True)
    _close(y_all, y_ref, torch.bfloat16)
    np.testing.assert_array_equal(_np(cache), so_ref)


def test_conv_decode_fp32_k3():
    M = make_mixer_inputs([1] * 33, H_qk=2, H_v=4, d_k=64, d_v=64, io_dtype=torch.float32,
                          seed=7)
    Md = M.to("cuda")
    w = Md.conv_weight[:, :3].contiguous()
    st = Md.conv_state[:, :2].contiguous()
    yd = gdn_conv1d_silu_decode(Md.x, w, None, st)
    assert gdn_sync_status() == 0
    y_ref, so_ref = oracle.conv1d_silu(M.x, M.conv_weight[:, :3], None, M.cu_seqlens.numpy(),
                                       M.conv_state[:, :2])
    _close(yd, y_ref, torch.float32)
    np.testing.assert_array_equal(_np(st), so_ref)


def test_conv_decode_cache_slots():
    """Caches in a pool of slots: each sequence slides its own entry; a padding entry
    (slot -1) gives zeros and touches nothing; unnamed entries come back bit for bit; a
    slot past the pool is reported."""
    N, pool_n = 5, 9
    M = make_mixer_inputs([1] * pool_n, H_qk=2, H_v=4, d_k=64, d_v=64, seed=13)
    slots = torch.tensor([7, 0, -1, 3, 8], dtype=torch.int32)
    Md = M.to("cuda")
    pool = Md.conv_state.clone()
    x = Md.x[:N].contiguous()
    y = gdn_conv1d_silu_decode(x, Md.conv_weight, Md.conv_bias, pool, slots.cuda())
    assert gdn_sync_status() == 0
    live = [n for n in range(N) if slots[n] >= 0]
    sl = [int(slots[n]) for n in live]
    y_ref, st_ref = oracle.conv1d_silu(M.x[live], M.conv_weight, M.conv_bias,
                                       np.arange(len(live) + 1), M.conv_state[sl])
    _close(y[live], y_ref, torch.bfloat16)
    np.testing.assert_array_equal(_np(pool[sl]), st_ref)
    assert torch.all(y[2] == 0)
    rest = sorted(set(range(pool_n)) - set(sl))
    assert torch.equal(pool[rest].cpu(), M.conv_state[rest])
    bad = torch.tensor([1, 9], dtype=torch.int32, device="cuda")
    gdn_conv1d_silu_decode(x[:2].contiguous(), Md.conv_weight, None, pool, bad)
    assert gdn_sync_status() == 7


def test_conv_bad_seqlens_reported():
    M = make_mixer_inputs(num_seqs=1, seq_len=40, H_qk=2, H_v=4, d_k=64, d_v=64, seed=8)
    Md = M.to("cuda")
    for bad in ([0, 30], [0, 50], [5, 40]):  # cu[N] < T, cu[N] > T, cu[0] > 0
        cu = torch.tensor(bad, dtype=torch.int32, device="cuda")
        gdn_conv1d_silu(Md.x, Md.conv_weight, None, cu, None)
        assert gdn_sync_status() == 6, bad
    assert gdn_sync_status() == 0


def test_conv_rejects_bad_arguments():
    M = make_mixer_inputs(num_seqs=1, seq_len=8, H_qk=2, H_v=4, d_k=64, d_v=64, seed=9).to("cuda")
    with pytest.raises(GDNError):
        gdn_conv1d_silu(M.x, M.conv_weight, None, M.cu_seqlens, None, out=M.x)
    with pytest.raises(GDNError):
        gdn_conv1d_silu(M.x[:, :12].contiguous(), M.conv_weight[:12].contiguous(), None,
                        M.cu_seqlens, None)


# ------------------------------------------------------------------ gated RMSNorm --

def test_rmsnorm_gated_35b_shape_bf16():
    """4096 tokens x 32 V heads x 128."""
    M = make_mixer_inputs(num_seqs=1, seq_len=4096, H_qk=1, H_v=32, d_k=8, d_v=128, seed=10)
    Md = M.to("cuda")
    y = gdn_rmsnorm_gated(Md.o, Md.z, Md.norm_weight, 1e-6)
    assert gdn_sync_status() == 0
    _close(y, oracle.rmsnorm_gated(M.o, M.z, M.norm_weight, 1e-6), torch.bfloat16)


@pytest.mark.parametrize("d", [64, 128])
def test_rmsnorm_gated_fp32_ragged_rows(d):
    """37 tokens x 3 heads: a row count that leaves the last block partly empty."""
    M = make_mixer_inputs(num_seqs=1, seq_len=37, H_qk=1, H_v=3, d_k=8, d_v=d,
                          io_dtype=torch.float32, seed=11)
    Md = M.to("cuda")
    y = gdn_rmsnorm_gated(Md.o, Md.z, Md.norm_weight, 1e-6)
    _close(y, oracle.rmsnorm_gated(M.o, M.z, M.norm_weight, 1e-6), torch.float32)


def test_rmsnorm_gated_in_place_and_degenerate_rows():
    """Output written over o; a zero row (y = 0), a huge row and a tiny row (eps decides)."""
    M = make_mixer_inputs(num_seqs=1, seq_len=9, H_qk=1, H_v=2, d_k=8, d_v=128, seed=12)
    o = M.o.clone()
    o[0, 0] = 0
    o[1, 0] = 3e4
    o[2, 1] = 1e-4
    od = o.cuda()
    y = gdn_rmsnorm_gated(od, M.z.cuda(), M.norm_weight.cuda(), 1e-6, out=od)
    assert y.data_ptr() == od.data_ptr()
    assert gdn_sync_status() == 0
    ref = oracle.rmsnorm_gated(o, M.z, M.norm_weight, 1e-6)
    _close(y, ref, torch.bfloat16)
    assert torch.all(y[0, 0] == 0)
