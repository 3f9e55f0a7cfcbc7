"""gdn_prefill_noalloc: the prefill for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc where they run the mixer (a runtime whose device
memory is owned by its own pool, a plugin given only its input and output buffers,
code where an allocation would block or synchronise the device), so they cannot hand
gdn_prefill a workspace. This entry point keeps that scratch in a fixed array inside
the library. The test calls it through the C ABI, twice in a row on different inputs
(the array keeps the previous call's contents), and checks each result against the
fp64 oracle and against gdn_prefill's, within the parity tolerance; once more at
exactly the array's capacity. It also checks, on the host, that a call one element
larger than the built-in scratch and calls with bad arguments are refused before
anything is launched, and that a call at exactly the capacity passes the size check.

This file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import oracle
from linear_attention_sequence_delta_b200 import gdn
from linear_attention_sequence_delta_b200.inputs import make_prefill_inputs
from tests.parity_util import TOL_BF16, TOL_FP32, rel_err

MAX_GATE_ELEMS = 1048576  # GDN_NOALLOC_MAX_GATE_ELEMS in include/gdn.h


def _fn():
    lib = gdn.load_library()
    f = lib.gdn_prefill_noalloc
    P, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    f.restype = ctypes.c_int
    f.argtypes = [P, P, P, i32, P, P, P, P, P, P, i32, i64, i32, i32, i32, i32, f32, P, P, P]
    return f


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call(P, o, Sf, scale=1.0):
    T, H_qk, d = P.q.shape
    H_v = P.v.shape[1]
    io = gdn.GDN_BF16 if P.q.dtype == torch.bfloat16 else gdn.GDN_FP32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return _fn()(_p(P.q), _p(P.k), _p(P.v), io, _p(P.a), _p(P.b), _p(P.A_log), _p(P.dt_bias),
                 _p(P.initial_state), _p(P.cu_seqlens), P.cu_seqlens.numel() - 1, T, H_qk, H_v,
                 d, d, scale, _p(o), _p(Sf), stream)


def test_refuses_more_than_the_builtin_scratch():
    # Rejected on the host before any CUDA call, so no GPU is needed.
    F = 0x7F0000000000
    v = ctypes.c_void_p
    H_v = 32
    T = MAX_GATE_ELEMS // H_v + 1
    st = _fn()(v(F), v(F), v(F), 0, v(F), v(F), v(F), v(F), None, v(F), 1, T, 16, H_v, 128, 128,
               1.0, v(F), None, None)
    assert st == 3  # GDN_ERR_WORKSPACE


def test_capacity_is_inclusive():
    # Exactly GDN_NOALLOC_MAX_GATE_ELEMS gate values pass the size check: with a
    # misaligned q the call then stops at the pointer checks that follow it
    # (GDN_ERR_INVALID_ARG, not GDN_ERR_WORKSPACE), still on the host.
    F = 0x7F0000000000
    v = ctypes.c_void_p
    for H_v in (4, 32):
        T = MAX_GATE_ELEMS // H_v
        st = _fn()(v(F + 8), v(F), v(F), 0, v(F), v(F), v(F), v(F), None, v(F), 1, T, 2,
                   H_v, 128, 128, 1.0, v(F), None, None)
        assert st == 1, H_v


@pytest.mark.parametrize("over,code", [
    (dict(io=7), 1),                       # not a dtype
    (dict(d=96), 2),                       # head size the library does not implement
    (dict(H_v=24), 1),                     # H_v not a multiple of H_qk
    (dict(N=-1), 1),
    (dict(N=0), 1),                        # tokens but no sequence
    (dict(scale=float("inf")), 1),
    (dict(cu=None), 1),
    (dict(q=0x7F0000000008), 1),           # not 16-byte aligned
    (dict(Sf=0x7F0000000004), 1),
    (dict(N=0, T=0), 0),                   # nothing to do: success, nothing launched
])
def test_host_checks(over, code):
    # Every case is decided on the host before any CUDA call, so no GPU is needed.
    F = 0x7F0000000000
    a = dict(io=0, N=1, T=256, H_qk=16, H_v=32, d=128, scale=1.0, cu=F, q=F, Sf=None)
    a.update(over)
    v = lambda p: None if p is None else ctypes.c_void_p(p)
    st = _fn()(v(a["q"]), v(F), v(F), a["io"], v(F), v(F), v(F), v(F), None, v(a["cu"]),
               a["N"], a["T"], a["H_qk"], a["H_v"], a["d"], a["d"], a["scale"], v(F),
               v(a["Sf"]), None)
    assert st == code


@pytest.mark.gpu
@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
def test_noalloc_matches_gdn_prefill_twice(io):
    tol = TOL_BF16 if io == torch.bfloat16 else TOL_FP32
    specs = [dict(lengths=[300, 1, 129], H_qk=2, H_v=4, d_k=128, d_v=128, state_std=0.05,
                  seed=31),
             dict(lengths=[64, 0, 517], H_qk=2, H_v=8, d_k=64, d_v=64, state_std=0.05,
                  seed=32)]
    for spec in specs:  # two calls in a row; the second reuses the array the first filled
        P = make_prefill_inputs(io_dtype=io, **spec).to("cuda")
        o_ref, S_ref = gdn.gdn_prefill(P.q, P.k, P.v, P.a, P.b, P.A_log, P.dt_bias,
                                       P.cu_seqlens, P.initial_state, scale=0.7)
        o = torch.full_like(o_ref, float("nan"))
        Sf = torch.full_like(S_ref, float("nan"))
        assert _call(P, o, Sf, scale=0.7) == 0
        assert gdn.gdn_sync_status() == 0
        assert rel_err(o, o_ref.float().cpu().numpy()) <= tol
        assert rel_err(Sf, S_ref.cpu().numpy()) <= tol
        Pc = P.to("cpu")
        o_or, S_or = oracle.forward(Pc.q, Pc.k, Pc.v, Pc.a, Pc.b, Pc.A_log, Pc.dt_bias,
                                    Pc.cu_seqlens.numpy(), Pc.initial_state, scale=0.7)
        assert rel_err(o, o_or) <= tol
        assert rel_err(Sf, S_or) <= tol


@pytest.mark.gpu
def test_noalloc_at_exactly_the_capacity():
    """T * H_v == GDN_NOALLOC_MAX_GATE_ELEMS: the beta half of the array ends at its
    last byte. 64 sequences of 4096 tokens, 4 V heads, d = 64, against the oracle."""
    P = make_prefill_inputs([4096] * 64, H_qk=2, H_v=4, d_k=64, d_v=64, state_std=0.05,
                            seed=33).to("cuda")
    assert P.q.shape[0] * P.v.shape[1] == MAX_GATE_ELEMS
    o = torch.full_like(P.v, float("nan"))
    Sf = torch.full_like(P.initial_state, float("nan"))
    assert _call(P, o, Sf) == 0
    assert gdn.gdn_sync_status() == 0
    Pc = P.to("cpu")
    o_or, S_or = oracle.forward(Pc.q, Pc.k, Pc.v, Pc.a, Pc.b, Pc.A_log, Pc.dt_bias,
                                Pc.cu_seqlens.numpy(), Pc.initial_state)
    assert rel_err(o, o_or) <= TOL_BF16
    assert rel_err(Sf, S_or) <= TOL_BF16
