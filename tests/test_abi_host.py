"""The C ABI on the host: exports, status strings, workspace sizing and argument
checks. No CUDA call is made here: every case is rejected before any launch,
so these run on a machine without a GPU. Pointer values are fake and aligned
(or deliberately misaligned); they are never dereferenced.
"""
import ctypes
import math
import os
import re

import pytest

from linear_attention_sequence_delta_b200 import build, gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return gdn.load_library()


def _declared():
    src = open(os.path.join(ROOT, "include", "gdn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    decl = _declared()
    assert set(decl) == set(gdn.EXPORTS)
    for name in decl:
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in gdn._STATUS.items():
        assert lib.gdn_status_string(code).decode() == name
    assert lib.gdn_status_string(99).decode() == "GDN_ERR_UNKNOWN"
    assert lib.gdn_version() >= 100


def test_workspace_size(lib):
    ws = lib.gdn_prefill_workspace_size
    a256 = lambda x: (x + 255) // 256 * 256
    # d = 128: chunk offsets and chain order (2 N + 1 int32), an 8-byte flag per record
    # and one 11,520-byte record per (chunk, V head), with at most ceil(T / 64) + N chunks
    tc = lambda N, ch, hv: a256((2 * N + 1) * 4) + a256(ch * hv * 8) + ch * hv * 11520
    assert ws(1, 4096, 16, 32, 128, 128) == tc(1, 64 + 1, 32)
    assert ws(4, 4 * 16384, 16, 64, 128, 128) == tc(4, 1024 + 4, 64)
    assert ws(64, 274156, 16, 32, 128, 128) == tc(64, (274156 + 63) // 64 + 64, 32)
    # never below the CUDA-core path's need (G and beta, fp32 [T, H_v] each)
    assert ws(1, 3, 1, 1, 128, 128) >= 2 * 256
    assert ws(1, 3, 1, 1, 64, 64) == 2 * 256  # each part rounded up to 256 bytes
    assert ws(0, 0, 16, 32, 128, 128) == 0
    assert ws(1, 10, 16, 24, 128, 128) == 0   # H_v % H_qk != 0
    assert ws(1, 10, 16, 32, 96, 96) == 0     # unsupported head dim
    assert ws(-1, 10, 16, 32, 128, 128) == 0


F = 0x7F0000000000  # fake, 256-byte aligned "device" address


def _prefill_args(**over):
    a = dict(q=F, k=F + 0x1000, v=F + 0x2000, io=gdn.GDN_BF16, a=F + 0x3000, b=F + 0x4000,
             A_log=F + 0x5000, dt_bias=F + 0x6000, S0=None, cu=F + 0x7000, N=1, T=128, H_qk=2,
             H_v=4, d_k=64, d_v=64, scale=1.0, o=F + 0x8000, Sf=None, ws=F + 0x10000,
             ws_bytes=1 << 20, stream=None)
    a.update(over)
    return a


def _call_prefill(lib, **over):
    a = _prefill_args(**over)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.gdn_prefill(v(a["q"]), v(a["k"]), v(a["v"]), a["io"], v(a["a"]), v(a["b"]),
                           v(a["A_log"]), v(a["dt_bias"]), v(a["S0"]), v(a["cu"]), a["N"], a["T"],
                           a["H_qk"], a["H_v"], a["d_k"], a["d_v"], a["scale"], v(a["o"]),
                           v(a["Sf"]), v(a["ws"]), a["ws_bytes"], v(a["stream"]))


@pytest.mark.parametrize("over,code", [
    (dict(io=7), 1),
    (dict(H_v=3), 1),                   # not a multiple of H_qk
    (dict(H_qk=0), 1),
    (dict(d_k=96, d_v=96), 2),
    (dict(d_k=64, d_v=128), 2),
    (dict(N=-1), 1),
    (dict(T=-5), 1),
    (dict(N=0, T=4), 1),
    (dict(scale=math.nan), 1),
    (dict(scale=math.inf), 1),
    (dict(q=None), 1),
    (dict(cu=None), 1),
    (dict(o=None), 1),
    (dict(A_log=None), 1),
    (dict(q=F + 8), 1),                  # misaligned
    (dict(o=F + 4), 1),
    (dict(S0=F + 2), 1),
    (dict(Sf=F + 12), 1),
    (dict(a=F + 2), 1),
    (dict(ws_bytes=100), 3),
    (dict(ws=None), 3),
    (dict(ws=F + 16), 3),               # workspace must be 256-byte aligned
])
def test_prefill_rejects(lib, over, code):
    assert _call_prefill(lib, **over) == code


def _call_prefill_ex(lib, opts, **over):
    a = _prefill_args(**over)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.gdn_prefill_ex(v(a["q"]), v(a["k"]), v(a["v"]), a["io"], v(a["a"]), v(a["b"]),
                              v(a["A_log"]), v(a["dt_bias"]), v(a["S0"]), v(a["cu"]), a["N"],
                              a["T"], a["H_qk"], a["H_v"], a["d_k"], a["d_v"], a["scale"],
                              v(a["o"]), v(a["Sf"]), v(a["ws"]), a["ws_bytes"],
                              None if opts is None else ctypes.byref(opts), v(a["stream"]))


@pytest.mark.parametrize("opts,over,code", [
    (dict(impl=5), {}, 1),                          # no such implementation
    (dict(impl=-1), {}, 1),
    (dict(fault=3), {}, 1),                         # no such fault
    (dict(fault=2), {}, 2),                         # index-check injection: debug build only
    (dict(wait_limit_cycles=-1), {}, 1),
    (dict(impl=2), {}, 2),                          # tensor cores forced, d = 64: unsupported
    (dict(impl=3), dict(io=gdn.GDN_FP32, d_k=128, d_v=128), 2),  # fp32 I/O
    (dict(impl=1), dict(ws_bytes=100), 3),          # the ordinary checks still apply
    (dict(impl=0), dict(N=0, T=0, q=None, k=None, v=None, o=None, ws=None, ws_bytes=0), 0),
])
def test_prefill_ex_rejects(lib, opts, over, code):
    """Per-call options are checked on the host, before any launch, like every argument."""
    o = gdn.PrefillOptions()
    for k_, v_ in opts.items():
        setattr(o, k_, v_)
    assert _call_prefill_ex(lib, o, **over) == code


@pytest.fixture(scope="module")
def debug_lib(lib):
    """libgdn_debug.so through a handle of its own (the module's library stays loaded),
    with the same argument and result types as the binding gives libgdn.so."""
    d = ctypes.CDLL(build.build(debug=True))
    for name in gdn.EXPORTS:
        f, g = getattr(lib, name), getattr(d, name)
        g.restype = f.restype
        if f.argtypes is not None:
            g.argtypes = f.argtypes
    return d


def test_debug_library_exports_and_flag(lib, debug_lib):
    for name in _declared():
        assert hasattr(debug_lib, name), name
    assert lib.gdn_debug_build() == 0
    assert debug_lib.gdn_debug_build() == 1
    assert debug_lib.gdn_status_string(8) == b"GDN_ERR_BAD_INDEX"


def test_debug_library_accepts_injection_option(debug_lib):
    """The debug build takes GDN_FAULT_BAD_INDEX and goes on to the ordinary checks (here
    a workspace too small: GDN_ERR_WORKSPACE, before any launch)."""
    o = gdn.PrefillOptions()
    o.fault = gdn.GDN_FAULT_BAD_INDEX
    assert _call_prefill_ex(debug_lib, o, ws_bytes=100) == 3
    o.fault = 3
    assert _call_prefill_ex(debug_lib, o) == 1


def test_prefill_ex_null_options_is_prefill(lib):
    for over in (dict(ws_bytes=100), dict(io=7), dict(N=0, T=0, q=None, k=None, v=None, o=None,
                                                     ws=None, ws_bytes=0)):
        assert _call_prefill_ex(lib, None, **over) == _call_prefill(lib, **over)


def test_prefill_empty_batch_is_noop(lib):
    # N = 0, T = 0: nothing to do, no CUDA call, success
    assert _call_prefill(lib, N=0, T=0, q=None, k=None, v=None, o=None, ws=None,
                         ws_bytes=0) == 0


def _call_decode(lib, **over):
    a = dict(q=F, k=F + 0x1000, v=F + 0x2000, io=gdn.GDN_BF16, a=F + 0x3000, b=F + 0x4000,
             A_log=F + 0x5000, dt_bias=F + 0x6000, S=F + 0x10000, N=8, H_qk=2, H_v=4, d_k=128,
             d_v=128, scale=1.0, o=F + 0x8000, stream=None)
    a.update(over)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.gdn_decode_step(v(a["q"]), v(a["k"]), v(a["v"]), a["io"], v(a["a"]), v(a["b"]),
                               v(a["A_log"]), v(a["dt_bias"]), v(a["S"]), a["N"], a["H_qk"],
                               a["H_v"], a["d_k"], a["d_v"], a["scale"], v(a["o"]),
                               v(a["stream"]))


@pytest.mark.parametrize("over,code", [
    (dict(io=-1), 1), (dict(H_v=5), 1), (dict(d_k=32, d_v=32), 2), (dict(N=-2), 1),
    (dict(S=None), 1), (dict(S=F + 4), 1), (dict(q=F + 2), 1), (dict(b=None), 1),
    (dict(scale=math.nan), 1),
])
def test_decode_rejects(lib, over, code):
    assert _call_decode(lib, **over) == code


def test_decode_bf16_state_rejects(lib):
    v = ctypes.c_void_p
    f = lib.gdn_decode_step_bf16_state
    args = lambda **o: dict(dict(q=F, k=F + 0x1000, vv=F + 0x2000, io=0, a=F + 0x3000,
                                 b=F + 0x4000, al=F + 0x5000, dt=F + 0x6000, S=F + 0x10000, N=8,
                                 hq=2, hv=4, dk=128, dv=128, sc=1.0, o=F + 0x8000), **o)
    p = lambda x: v(x) if x else None
    call = lambda a: f(p(a["q"]), p(a["k"]), p(a["vv"]), a["io"], p(a["a"]), p(a["b"]),
                       p(a["al"]), p(a["dt"]), p(a["S"]), a["N"], a["hq"], a["hv"], a["dk"],
                       a["dv"], a["sc"], p(a["o"]), None)
    assert call(args(io=3)) == 1
    assert call(args(hv=5)) == 1
    assert call(args(dk=96, dv=96)) == 2
    assert call(args(S=None)) == 1
    assert call(args(S=F + 0x10008)) == 1
    assert call(args(sc=math.nan)) == 1
    assert call(args(N=0)) == 0


def test_decode_zero_sequences_is_noop(lib):
    assert _call_decode(lib, N=0) == 0


def test_gates_rejects(lib):
    v = ctypes.c_void_p
    g = lib.gdn_gates
    assert g(v(F), v(F), v(F), v(F), v(F), -1, 4, 4, v(F), None, None, None) == 1
    assert g(v(F), v(F), v(F), v(F), v(F), 1, 4, 0, v(F), None, None, None) == 1
    assert g(None, v(F), v(F), v(F), v(F), 1, 4, 4, v(F), None, None, None) == 1
    assert g(v(F + 2), v(F), v(F), v(F), v(F), 1, 4, 4, v(F), None, None, None) == 1
    # nothing asked for: success without a launch
    assert g(v(F), v(F), v(F), v(F), v(F), 1, 4, 4, None, None, None, None) == 0


def _call_conv(lib, **over):
    a = dict(x=F, io=gdn.GDN_BF16, w=F + 0x1000, bias=None, sin=None, cu=F + 0x2000, N=2, T=64,
             C=256, K=4, y=F + 0x8000, sout=None, stream=None)
    a.update(over)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.gdn_conv1d_silu(v(a["x"]), a["io"], v(a["w"]), v(a["bias"]), v(a["sin"]),
                               v(a["cu"]), a["N"], a["T"], a["C"], a["K"], v(a["y"]),
                               v(a["sout"]), v(a["stream"]))


@pytest.mark.parametrize("over,code", [
    (dict(io=3), 1), (dict(N=-1), 1), (dict(T=-1), 1), (dict(C=0), 1), (dict(N=0, T=8), 1),
    (dict(K=1), 2), (dict(K=5), 2), (dict(C=260), 2),
    (dict(x=None), 1), (dict(w=None), 1), (dict(cu=None), 1), (dict(y=None), 1),
    (dict(x=F + 8), 1), (dict(y=F + 4), 1), (dict(w=F + 4), 1), (dict(sin=F + 2), 1),
    (dict(sout=F + 8), 1), (dict(bias=F + 2), 1), (dict(cu=F + 2), 1),
    (dict(y=F), 1),                     # in place is refused: the window reads neighbours
])
def test_conv1d_rejects(lib, over, code):
    assert _call_conv(lib, **over) == code


def test_conv1d_noops(lib):
    assert _call_conv(lib, N=0, T=0, x=None, y=None) == 0
    assert _call_conv(lib, T=0, y=None) == 0          # no tokens, no cache asked for


def test_conv1d_decode_rejects(lib):
    v = ctypes.c_void_p
    d = lib.gdn_conv1d_silu_decode
    ok = lambda **o: dict(dict(x=F, io=0, w=F + 0x1000, b=None, st=F + 0x2000, sl=None, ns=4,
                               N=4, C=64, K=4, y=F + 0x3000), **o)
    p = lambda x: v(x) if x else None
    call = lambda a: d(p(a["x"]), a["io"], p(a["w"]), p(a["b"]), p(a["st"]), p(a["sl"]),
                       a["ns"], a["N"], a["C"], a["K"], p(a["y"]), None)
    assert call(ok(io=2)) == 1
    assert call(ok(N=-1)) == 1
    assert call(ok(ns=-1)) == 1
    assert call(ok(ns=3)) == 1            # identity slots need N cache entries
    assert call(ok(K=6)) == 2
    assert call(ok(C=12)) == 2
    assert call(ok(st=None)) == 1
    assert call(ok(st=F + 0x2004)) == 1
    assert call(ok(b=F + 1)) == 1
    assert call(ok(sl=F + 0x4002, ns=2)) == 1
    assert call(ok(N=0)) == 0


def test_rmsnorm_gated_rejects(lib):
    v = ctypes.c_void_p
    r = lib.gdn_rmsnorm_gated
    assert r(v(F), v(F + 0x100), 5, v(F + 0x200), 1e-6, 4, 128, v(F + 0x300), None) == 1
    assert r(v(F), v(F + 0x100), 0, v(F + 0x200), 1e-6, -1, 128, v(F + 0x300), None) == 1
    assert r(v(F), v(F + 0x100), 0, v(F + 0x200), -1.0, 4, 128, v(F + 0x300), None) == 1
    assert r(v(F), v(F + 0x100), 0, v(F + 0x200), math.nan, 4, 128, v(F + 0x300), None) == 1
    assert r(v(F), v(F + 0x100), 0, v(F + 0x200), 1e-6, 4, 96, v(F + 0x300), None) == 2
    assert r(None, v(F + 0x100), 0, v(F + 0x200), 1e-6, 4, 128, v(F + 0x300), None) == 1
    assert r(v(F), v(F + 0x100), 0, v(F + 0x204), 1e-6, 4, 128, v(F + 0x300), None) == 1
    assert r(v(F + 8), v(F + 0x100), 0, v(F + 0x200), 1e-6, 4, 128, v(F + 0x300), None) == 1
    assert r(None, None, 0, None, 1e-6, 0, 128, None, None) == 0


def _call_slots(lib, **over):
    a = dict(q=F, k=F + 0x1000, v=F + 0x2000, io=gdn.GDN_BF16, a=F + 0x3000, b=F + 0x4000,
             A_log=F + 0x5000, dt_bias=F + 0x6000, pool=F + 0x10000, slots=F + 0x7000, ns=8,
             N=4, L=2, H_qk=2, H_v=4, d_k=128, d_v=128, scale=1.0, o=F + 0x8000, inter=None)
    a.update(over)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.gdn_decode_slots(v(a["q"]), v(a["k"]), v(a["v"]), a["io"], v(a["a"]), v(a["b"]),
                                v(a["A_log"]), v(a["dt_bias"]), v(a["pool"]), v(a["slots"]),
                                a["ns"], a["N"], a["L"], a["H_qk"], a["H_v"], a["d_k"], a["d_v"],
                                a["scale"], v(a["o"]), v(a["inter"]), None)


@pytest.mark.parametrize("over,code", [
    (dict(io=2), 1), (dict(N=-1), 1), (dict(ns=-1), 1), (dict(L=0), 2), (dict(L=17), 2),
    (dict(H_v=5), 1), (dict(d_k=32, d_v=32), 2), (dict(scale=math.inf), 1),
    (dict(slots=None, ns=3), 1),        # identity slots need a pool of at least N states
    (dict(q=None), 1), (dict(o=None), 1), (dict(pool=None), 1),
    (dict(pool=F + 8), 1), (dict(inter=F + 4), 1), (dict(slots=F + 2), 1), (dict(a=F + 1), 1),
])
def test_decode_slots_rejects(lib, over, code):
    assert _call_slots(lib, **over) == code


def test_prefill_slots_rejects(lib):
    v = ctypes.c_void_p
    f = lib.gdn_prefill_slots
    base = dict(q=F, k=F + 0x1000, vv=F + 0x2000, io=0, a=F + 0x3000, b=F + 0x4000,
                al=F + 0x5000, dt=F + 0x6000, pool=F + 0x10000, sl=F + 0x7000, hi=None, ns=4,
                cu=F + 0x7100, N=2, T=128, hq=2, hv=4, dk=128, dv=128, sc=1.0, o=F + 0x8000,
                ws=F + 0x100000, wsb=1 << 30)
    p = lambda x: v(x) if x else None
    call = lambda **o: (lambda a: f(p(a["q"]), p(a["k"]), p(a["vv"]), a["io"], p(a["a"]),
                                    p(a["b"]), p(a["al"]), p(a["dt"]), p(a["pool"]), p(a["sl"]),
                                    p(a["hi"]), a["ns"], p(a["cu"]), a["N"], a["T"], a["hq"],
                                    a["hv"], a["dk"], a["dv"], a["sc"], p(a["o"]), p(a["ws"]),
                                    a["wsb"], None))(dict(base, **o))
    assert call(sl=None) == 1
    assert call(pool=None) == 1
    assert call(ns=-1) == 1
    assert call(sl=F + 0x7002) == 1
    assert call(hi=F + 0x7203) == 1
    assert call(pool=F + 0x10004) == 1   # the pool is the initial / final state array
    assert call(io=5) == 1
    assert call(wsb=10) == 3
    assert call(N=0, T=0, sl=None, pool=None) == 0


def test_decode_slots_noop(lib):
    assert _call_slots(lib, N=0) == 0
    assert _call_slots(lib, N=0, slots=None, ns=0, pool=None) == 0


def test_binding_fails_loudly_without_library(tmp_path):
    saved = gdn._lib
    try:
        gdn._lib = None
        with pytest.raises(RuntimeError, match="libgdn.so not found"):
            gdn.load_library(str(tmp_path / "missing.so"))
    finally:
        gdn._lib = saved


def test_timer_host_checks(lib):
    """The timer calls reject null handles without touching the GPU."""
    ms = (ctypes.c_float * 4)()
    assert lib.gdn_timer_read(None, ms, 4) == -1
    assert lib.gdn_timer_kernel_name(None, 0) is None
    lib.gdn_timer_destroy(None)  # ignored


def _call_mixer(lib, **over):
    a = dict(x=F, io=gdn.GDN_BF16, w=F + 0x1000, bias=None, cin=None, cout=None, K=4,
             a=F + 0x3000, b=F + 0x4000, A_log=F + 0x5000, dt_bias=F + 0x6000, S0=None,
             cu=F + 0x7000, N=1, T=128, H_qk=2, H_v=4, d=64, scale=1.0, z=F + 0x8000,
             nw=F + 0x9000, eps=1e-6, y=F + 0xA000, Sf=None, ws=F + 0x10000, ws_bytes=1 << 30,
             opts=None)
    a.update(over)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.gdn_mixer_prefill(v(a["x"]), a["io"], v(a["w"]), v(a["bias"]), v(a["cin"]),
                                 v(a["cout"]), a["K"], v(a["a"]), v(a["b"]), v(a["A_log"]),
                                 v(a["dt_bias"]), v(a["S0"]), v(a["cu"]), a["N"], a["T"],
                                 a["H_qk"], a["H_v"], a["d"], a["d"], a["scale"], v(a["z"]),
                                 v(a["nw"]), a["eps"], v(a["y"]), v(a["Sf"]), v(a["ws"]),
                                 a["ws_bytes"], a["opts"], None)


@pytest.mark.parametrize("over,code", [
    (dict(io=3), 1),
    (dict(K=5), 2), (dict(K=1), 2),
    (dict(d=96), 2),
    (dict(H_v=3), 1),
    (dict(eps=-1.0), 1), (dict(eps=math.inf), 1), (dict(scale=math.nan), 1),
    (dict(N=0, T=5), 1),
    (dict(x=None), 1), (dict(z=None), 1), (dict(y=None), 1), (dict(w=None), 1),
    (dict(nw=None), 1), (dict(cu=None), 1),
    (dict(y=F), 1),                     # y must not be x
    (dict(y=F + 0x8000), 1),            # nor z
    (dict(nw=F + 4), 1), (dict(cout=F + 8), 1), (dict(x=F + 2), 1), (dict(bias=F + 2), 1),
    (dict(ws_bytes=1000), 3), (dict(ws=F + 0x10010), 3), (dict(ws=None), 3),
    (dict(N=0, T=0), 0),                # nothing to do
])
def test_mixer_prefill_rejects(lib, over, code):
    assert _call_mixer(lib, **over) == code


def test_mixer_workspace_size(lib):
    f = lib.gdn_mixer_prefill_workspace_size
    pre = lib.gdn_prefill_workspace_size(1, 4096, 16, 32, 128, 128)
    conv_dim = (2 * 16 + 32) * 128
    assert f(1, 4096, 16, 32, 128, 128, gdn.GDN_BF16) == 4096 * conv_dim * 2 + pre
    assert f(1, 4096, 16, 32, 128, 128, gdn.GDN_FP32) == 4096 * conv_dim * 4 + pre
    assert f(1, 4096, 16, 32, 128, 128, 7) == 0
    assert f(1, 10, 16, 24, 128, 128, gdn.GDN_BF16) == 0
