"""Python binding of libgdn.so (argument marshalling only).

Every step of the computation runs in the library's CUDA kernels; this module
only checks tensor metadata, allocates outputs/workspace through torch, and
passes raw pointers and the current CUDA stream across the C ABI declared in
include/gdn.h. There is no fallback: if the library is missing or cannot be
loaded, every call raises.

The calls keep the C names:
  gdn_gates(a, b, A_log, dt_bias, cu_seqlens, ...)
  gdn_prefill(q, k, v, a, b, A_log, dt_bias, cu_seqlens, initial_state=None, ...)
  gdn_decode_step(q, k, v, a, b, A_log, dt_bias, state, ...)
and the steps around the delta rule in the mixer:
  gdn_conv1d_silu(x, weight, bias, cu_seqlens, conv_state_in=None, ...)
  gdn_conv1d_silu_decode(x, weight, bias, conv_state, ...)
  gdn_rmsnorm_gated(o, z, weight, eps=1e-6, ...)
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
DEFAULT_LIB_PATH = os.path.join(_HERE, "libgdn.so")
DEBUG_LIB_PATH = os.path.join(_HERE, "libgdn_debug.so")  # kernels with index checks
# The library a process loads: libgdn.so, or the file GDN_LIBRARY names (for instance
# libgdn_debug.so, the same ABI with the kernels' index checks compiled in).
LIB_PATH = os.environ.get("GDN_LIBRARY") or DEFAULT_LIB_PATH

GDN_BF16, GDN_FP32 = 0, 1
_STATUS = {0: "GDN_OK", 1: "GDN_ERR_INVALID_ARG", 2: "GDN_ERR_UNSUPPORTED", 3: "GDN_ERR_WORKSPACE",
           4: "GDN_ERR_CUDA", 5: "GDN_ERR_TIMEOUT", 6: "GDN_ERR_BAD_SEQLENS",
           7: "GDN_ERR_BAD_SLOT", 8: "GDN_ERR_BAD_INDEX"}

# Every symbol include/gdn.h declares (the tests check the library exports them all).
EXPORTS = ["gdn_status_string", "gdn_version", "gdn_prefill_workspace_size", "gdn_gates",
           "gdn_prefill", "gdn_prefill_ex", "gdn_decode_step", "gdn_sync_status",
           "gdn_prefill_noalloc", "gdn_timer_create", "gdn_timer_destroy", "gdn_timer_read",
           "gdn_timer_kernel_name", "gdn_conv1d_silu", "gdn_conv1d_silu_decode",
           "gdn_rmsnorm_gated", "gdn_decode_slots", "gdn_decode_step_bf16_state",
           "gdn_prefill_slots", "gdn_prefill_slots_ex", "gdn_mixer_prefill",
           "gdn_mixer_prefill_workspace_size", "gdn_debug_build", "gdn_debug_bad_index_site"]
GDN_IMPL_AUTO, GDN_IMPL_CUDA_CORE, GDN_IMPL_TENSOR_CORE, GDN_IMPL_TENSOR_CORE_SPLIT = 0, 1, 2, 3
GDN_IMPL_TENSOR_CORE_WHOLE_ROWS = 4
GDN_FAULT_NONE, GDN_FAULT_WITHHOLD_RECORDS, GDN_FAULT_BAD_INDEX = 0, 1, 2


class PrefillOptions(ctypes.Structure):
    """gdn_prefill_options of include/gdn.h (per-call implementation choice, fault
    injection, wait limit, kernel timer)."""
    _fields_ = [("impl", ctypes.c_int32), ("fault", ctypes.c_int32),
                ("wait_limit_cycles", ctypes.c_int64), ("timer", ctypes.c_void_p)]


class GDNError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_STATUS.get(status, status)}")


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libgdn.so (built by `python -m linear_attention_sequence_delta_b200.build`)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libgdn.so not found at {path}; build it with "
                           "`python -m linear_attention_sequence_delta_b200.build`")
    lib = ctypes.CDLL(path)
    P, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                            ctypes.c_size_t)
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_status_string.argtypes = [ctypes.c_int]
    lib.gdn_version.restype = ctypes.c_int
    lib.gdn_prefill_workspace_size.restype = sz
    lib.gdn_prefill_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32]
    lib.gdn_gates.restype = ctypes.c_int
    lib.gdn_gates.argtypes = [P, P, P, P, P, i32, i64, i32, P, P, P, P]
    lib.gdn_prefill.restype = ctypes.c_int
    lib.gdn_prefill.argtypes = [P, P, P, i32, P, P, P, P, P, P, i32, i64, i32, i32, i32, i32, f32,
                                P, P, P, sz, P]
    lib.gdn_decode_step.restype = ctypes.c_int
    lib.gdn_decode_step.argtypes = [P, P, P, i32, P, P, P, P, P, i32, i32, i32, i32, i32, f32, P,
                                    P]
    lib.gdn_sync_status.restype = ctypes.c_int
    lib.gdn_sync_status.argtypes = [P]
    lib.gdn_debug_build.restype = ctypes.c_int
    lib.gdn_debug_build.argtypes = []
    lib.gdn_debug_bad_index_site.restype = ctypes.c_int
    lib.gdn_debug_bad_index_site.argtypes = [P]
    lib.gdn_prefill_ex.restype = ctypes.c_int
    lib.gdn_prefill_ex.argtypes = [P, P, P, i32, P, P, P, P, P, P, i32, i64, i32, i32, i32, i32,
                                   f32, P, P, P, sz, P, P]
    lib.gdn_prefill_slots_ex.restype = ctypes.c_int
    lib.gdn_prefill_slots_ex.argtypes = [P, P, P, i32, P, P, P, P, P, P, P, i32, P, i32, i64,
                                         i32, i32, i32, i32, f32, P, P, sz, P, P]
    lib.gdn_timer_create.restype = P
    lib.gdn_timer_create.argtypes = []
    lib.gdn_timer_destroy.restype = None
    lib.gdn_timer_destroy.argtypes = [P]
    lib.gdn_timer_read.restype = ctypes.c_int
    lib.gdn_timer_read.argtypes = [P, P, i32]
    lib.gdn_timer_kernel_name.restype = ctypes.c_char_p
    lib.gdn_timer_kernel_name.argtypes = [P, i32]
    lib.gdn_conv1d_silu.restype = ctypes.c_int
    lib.gdn_conv1d_silu.argtypes = [P, i32, P, P, P, P, i32, i64, i32, i32, P, P, P]
    lib.gdn_conv1d_silu_decode.restype = ctypes.c_int
    lib.gdn_conv1d_silu_decode.argtypes = [P, i32, P, P, P, P, i32, i32, i32, i32, P, P]
    lib.gdn_prefill_slots.restype = ctypes.c_int
    lib.gdn_prefill_slots.argtypes = [P, P, P, i32, P, P, P, P, P, P, P, i32, P, i32, i64, i32,
                                      i32, i32, i32, f32, P, P, sz, P]
    lib.gdn_decode_step_bf16_state.restype = ctypes.c_int
    lib.gdn_decode_step_bf16_state.argtypes = [P, P, P, i32, P, P, P, P, P, i32, i32, i32, i32,
                                               i32, f32, P, P]
    lib.gdn_decode_slots.restype = ctypes.c_int
    lib.gdn_decode_slots.argtypes = [P, P, P, i32, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32,
                                     i32, f32, P, P, P]
    lib.gdn_mixer_prefill_workspace_size.restype = sz
    lib.gdn_mixer_prefill_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32, i32]
    lib.gdn_mixer_prefill.restype = ctypes.c_int
    lib.gdn_mixer_prefill.argtypes = [P, i32, P, P, P, P, i32, P, P, P, P, P, P, i32, i64, i32,
                                      i32, i32, i32, f32, P, P, f32, P, P, P, sz, P, P]
    lib.gdn_rmsnorm_gated.restype = ctypes.c_int
    lib.gdn_rmsnorm_gated.argtypes = [P, P, i32, P, f32, i64, i32, P, P]
    _lib = lib
    return lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _io_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_FP32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _check(status: int, where: str):
    if status != 0:
        raise GDNError(status, where)


def _need_cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("all tensors must be CUDA tensors")
            if not t.is_contiguous():
                raise ValueError("all tensors must be contiguous")


def workspace_size(num_seqs, total_tokens, H_qk, H_v, d_k, d_v) -> int:
    return int(load_library().gdn_prefill_workspace_size(num_seqs, total_tokens, H_qk, H_v, d_k,
                                                         d_v))


def gdn_gates(a, b, A_log, dt_bias, cu_seqlens, *, want_cumsum=True, want_g=True,
              want_beta=True) -> Tuple[Optional[torch.Tensor], ...]:
    """Returns (g_chunk_cumsum, g, beta), fp32 [T, H_v] each (None where not asked for)."""
    lib = load_library()
    _need_cuda(a, b, A_log, dt_bias, cu_seqlens)
    T, H_v = a.shape
    mk = lambda w: torch.empty((T, H_v), device=a.device, dtype=torch.float32) if w else None
    G, g, beta = mk(want_cumsum), mk(want_g), mk(want_beta)
    st = lib.gdn_gates(_ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias), _ptr(cu_seqlens),
                       cu_seqlens.numel() - 1, T, H_v, _ptr(G), _ptr(g), _ptr(beta),
                       _stream(a.device))
    _check(st, "gdn_gates")
    return G, g, beta


class Timer:
    """A gdn_timer: CUDA events around every kernel of the calls it is passed to."""

    def __init__(self):
        self._lib = load_library()
        self._t = self._lib.gdn_timer_create()
        if not self._t:
            raise GDNError(4, "gdn_timer_create")
        # held here so that close() needs no module global (at interpreter exit those
        # may already be gone when the finaliser runs)
        self._handle = ctypes.c_void_p(self._t)
        self._destroy = self._lib.gdn_timer_destroy

    def times(self) -> list:
        """[(kernel name, milliseconds)] of the most recent call made with this timer
        (waits for its events)."""
        ms = (ctypes.c_float * 8)()
        n = int(self._lib.gdn_timer_read(ctypes.c_void_p(self._t), ms, 8))
        if n < 0:
            raise GDNError(-n, "gdn_timer_read")
        return [(self._lib.gdn_timer_kernel_name(ctypes.c_void_p(self._t), i).decode(),
                 float(ms[i])) for i in range(min(n, 8))]

    def close(self):
        if getattr(self, "_t", None):
            self._destroy(self._handle)
            self._t = None

    def __del__(self):
        self.close()


def _options(impl, fault, wait_limit_cycles, timer):
    if impl == GDN_IMPL_AUTO and fault == GDN_FAULT_NONE and not wait_limit_cycles and \
            timer is None:
        return None
    return ctypes.byref(PrefillOptions(int(impl), int(fault), int(wait_limit_cycles),
                                       None if timer is None else timer._t))


def gdn_prefill(q, k, v, a, b, A_log, dt_bias, cu_seqlens, initial_state=None, *,
                scale: float = 1.0, output_final_state: bool = True, out=None,
                final_state=None, workspace=None, impl: int = GDN_IMPL_AUTO,
                timer: Optional[Timer] = None, fault: int = GDN_FAULT_NONE,
                wait_limit_cycles: int = 0):
    """Chunked prefill over a packed batch. Returns (o, final_state or None).

    q, k [T, H_qk, d_k]; v [T, H_v, d_v] (bf16 or fp32, all the same);
    a, b [T, H_v] fp32; A_log, dt_bias [H_v] fp32; cu_seqlens int32 [N+1];
    initial_state [N, H_v, d_v, d_k] fp32 or None. impl, timer, fault and
    wait_limit_cycles are gdn_prefill_options (gdn_prefill_ex).
    """
    lib = load_library()
    _need_cuda(q, k, v, a, b, A_log, dt_bias, cu_seqlens, initial_state, out, final_state,
               workspace)
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k and v must share one dtype")
    io = _io_dtype(q)
    T, H_qk, d_k = q.shape
    _, H_v, d_v = v.shape
    N = cu_seqlens.numel() - 1
    o = out if out is not None else torch.empty((T, H_v, d_v), device=q.device, dtype=q.dtype)
    if output_final_state and final_state is None:
        final_state = torch.empty((N, H_v, d_v, d_k), device=q.device, dtype=torch.float32)
    if not output_final_state:
        final_state = None
    need = lib.gdn_prefill_workspace_size(N, T, H_qk, H_v, d_k, d_v)
    if workspace is None:
        workspace = torch.empty((max(int(need), 1),), device=q.device, dtype=torch.uint8)
    opts = _options(impl, fault, wait_limit_cycles, timer)
    args = (_ptr(q), _ptr(k), _ptr(v), io, _ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias),
            _ptr(initial_state), _ptr(cu_seqlens), N, T, H_qk, H_v, d_k, d_v, float(scale),
            _ptr(o), _ptr(final_state), _ptr(workspace), workspace.numel())
    if opts is None:
        st = lib.gdn_prefill(*args, _stream(q.device))
    else:
        st = lib.gdn_prefill_ex(*args, opts, _stream(q.device))
    _check(st, "gdn_prefill")
    return o, final_state


def gdn_prefill_slots(q, k, v, a, b, A_log, dt_bias, cu_seqlens, state_pool, state_slots,
                      has_initial_state=None, *, scale: float = 1.0, out=None, workspace=None,
                      impl: int = GDN_IMPL_AUTO):
    """gdn_prefill with the states in a pool: sequence n starts from state_pool[slot]
    (or zeros where has_initial_state[n] == 0) and its final state replaces it.
    state_pool [num_slots, H_v, d_v, d_k] fp32; state_slots, has_initial_state int32 [N]."""
    lib = load_library()
    _need_cuda(q, k, v, a, b, A_log, dt_bias, cu_seqlens, state_pool, state_slots,
               has_initial_state, out, workspace)
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k and v must share one dtype")
    for t in (state_slots, has_initial_state):
        if t is not None and t.dtype != torch.int32:
            raise TypeError("state_slots and has_initial_state must be int32")
    io = _io_dtype(q)
    T, H_qk, d_k = q.shape
    _, H_v, d_v = v.shape
    N = cu_seqlens.numel() - 1
    o = out if out is not None else torch.empty((T, H_v, d_v), device=q.device, dtype=q.dtype)
    need = lib.gdn_prefill_workspace_size(N, T, H_qk, H_v, d_k, d_v)
    if workspace is None:
        workspace = torch.empty((max(int(need), 1),), device=q.device, dtype=torch.uint8)
    args = (_ptr(q), _ptr(k), _ptr(v), io, _ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias),
            _ptr(state_pool), _ptr(state_slots), _ptr(has_initial_state), state_pool.shape[0],
            _ptr(cu_seqlens), N, T, H_qk, H_v, d_k, d_v, float(scale), _ptr(o), _ptr(workspace),
            workspace.numel())
    opts = _options(impl, GDN_FAULT_NONE, 0, None)
    if opts is None:
        st = lib.gdn_prefill_slots(*args, _stream(q.device))
    else:
        st = lib.gdn_prefill_slots_ex(*args, opts, _stream(q.device))
    _check(st, "gdn_prefill_slots")
    return o


def gdn_decode_step(q, k, v, a, b, A_log, dt_bias, state, *, scale: float = 1.0, out=None):
    """One token per sequence; `state` [N, H_v, d_v, d_k] fp32 is updated in place.

    q, k [N, H_qk, d_k]; v [N, H_v, d_v]; a, b [N, H_v]. Returns o [N, H_v, d_v].
    """
    lib = load_library()
    _need_cuda(q, k, v, a, b, A_log, dt_bias, state, out)
    io = _io_dtype(q)
    N, H_qk, d_k = q.shape
    _, H_v, d_v = v.shape
    o = out if out is not None else torch.empty((N, H_v, d_v), device=q.device, dtype=q.dtype)
    st = lib.gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), io, _ptr(a), _ptr(b), _ptr(A_log),
                             _ptr(dt_bias), _ptr(state), N, H_qk, H_v, d_k, d_v, float(scale),
                             _ptr(o), _stream(q.device))
    _check(st, "gdn_decode_step")
    return o


def gdn_decode_step_bf16_state(q, k, v, a, b, A_log, dt_bias, state, *, scale: float = 1.0,
                               out=None):
    """gdn_decode_step with a bf16 state [N, H_v, d_v, d_k] updated in place. Returns o."""
    lib = load_library()
    _need_cuda(q, k, v, a, b, A_log, dt_bias, state, out)
    if state.dtype != torch.bfloat16:
        raise TypeError("state must be bfloat16")
    io = _io_dtype(q)
    N, H_qk, d_k = q.shape
    _, H_v, d_v = v.shape
    o = out if out is not None else torch.empty((N, H_v, d_v), device=q.device, dtype=q.dtype)
    st = lib.gdn_decode_step_bf16_state(_ptr(q), _ptr(k), _ptr(v), io, _ptr(a), _ptr(b),
                                        _ptr(A_log), _ptr(dt_bias), _ptr(state), N, H_qk, H_v,
                                        d_k, d_v, float(scale), _ptr(o), _stream(q.device))
    _check(st, "gdn_decode_step_bf16_state")
    return o


def gdn_decode_slots(q, k, v, a, b, A_log, dt_bias, state_pool, state_slots=None, *,
                     scale: float = 1.0, out=None, intermediate_states=None,
                     want_intermediate: bool = False):
    """L tokens per sequence from a pool of states; the pool is updated in place.

    q, k [N, L, H_qk, d_k]; v [N, L, H_v, d_v]; a, b [N, L, H_v] fp32;
    state_pool [num_slots, H_v, d_v, d_k] fp32; state_slots int32 [N] or None (slot n).
    Returns (o [N, L, H_v, d_v], intermediate states [N, L, H_v, d_v, d_k] or None).
    """
    lib = load_library()
    _need_cuda(q, k, v, a, b, A_log, dt_bias, state_pool, state_slots, out, intermediate_states)
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k and v must share one dtype")
    if state_slots is not None and state_slots.dtype != torch.int32:
        raise TypeError("state_slots must be int32")
    io = _io_dtype(q)
    N, L, H_qk, d_k = q.shape
    H_v, d_v = v.shape[2], v.shape[3]
    o = out if out is not None else torch.empty((N, L, H_v, d_v), device=q.device, dtype=q.dtype)
    if want_intermediate and intermediate_states is None:
        intermediate_states = torch.empty((N, L, H_v, d_v, d_k), device=q.device,
                                          dtype=torch.float32)
    st = lib.gdn_decode_slots(_ptr(q), _ptr(k), _ptr(v), io, _ptr(a), _ptr(b), _ptr(A_log),
                              _ptr(dt_bias), _ptr(state_pool), _ptr(state_slots),
                              state_pool.shape[0], N, L, H_qk, H_v, d_k, d_v, float(scale),
                              _ptr(o), _ptr(intermediate_states), _stream(q.device))
    _check(st, "gdn_decode_slots")
    return o, intermediate_states


def gdn_sync_status(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device status word."""
    lib = load_library()
    return int(lib.gdn_sync_status(_stream(device)))


def debug_build() -> bool:
    """True when the loaded library is libgdn_debug.so (kernels with index checks)."""
    return bool(load_library().gdn_debug_build())


def debug_bad_index_site(device=None) -> int:
    """Synchronise the current stream; return (and clear) the source line of the first
    failed index check of the debug build since the last call (0: none)."""
    r = int(load_library().gdn_debug_bad_index_site(_stream(device)))
    if r < 0:
        raise GDNError(-r, "gdn_debug_bad_index_site")
    return r


def gdn_conv1d_silu(x, weight, bias, cu_seqlens, conv_state_in=None, *, want_state=True,
                    out=None, conv_state_out=None):
    """Causal depthwise conv1d + SiLU over a packed batch. Returns (y, conv_state_out or None).

    x [T, C] (bf16 or fp32); weight [C, K] fp32; bias [C] fp32 or None; cu_seqlens int32
    [N+1]; conv_state_in [N, K-1, C] (x's dtype) or None (zeros). conv_state_out may be
    conv_state_in (updated in place).
    """
    lib = load_library()
    _need_cuda(x, weight, bias, cu_seqlens, conv_state_in, out, conv_state_out)
    io = _io_dtype(x)
    T, C = x.shape
    K = weight.shape[1]
    N = cu_seqlens.numel() - 1
    y = out if out is not None else torch.empty_like(x)
    if want_state and conv_state_out is None:
        conv_state_out = torch.empty((N, K - 1, C), device=x.device, dtype=x.dtype)
    if not want_state:
        conv_state_out = None
    st = lib.gdn_conv1d_silu(_ptr(x), io, _ptr(weight), _ptr(bias), _ptr(conv_state_in),
                             _ptr(cu_seqlens), N, T, C, K, _ptr(y), _ptr(conv_state_out),
                             _stream(x.device))
    _check(st, "gdn_conv1d_silu")
    return y, conv_state_out


def gdn_conv1d_silu_decode(x, weight, bias, conv_state, cache_slots=None, *, out=None):
    """One token per sequence: x [N, C]; conv_state [num_slots, K-1, C] (a pool of caches)
    slides in place; cache_slots int32 [N] or None (entry n). Returns y [N, C]."""
    lib = load_library()
    _need_cuda(x, weight, bias, conv_state, cache_slots, out)
    if cache_slots is not None and cache_slots.dtype != torch.int32:
        raise TypeError("cache_slots must be int32")
    io = _io_dtype(x)
    N, C = x.shape
    K = weight.shape[1]
    y = out if out is not None else torch.empty_like(x)
    st = lib.gdn_conv1d_silu_decode(_ptr(x), io, _ptr(weight), _ptr(bias), _ptr(conv_state),
                                    _ptr(cache_slots), conv_state.shape[0], N, C, K, _ptr(y),
                                    _stream(x.device))
    _check(st, "gdn_conv1d_silu_decode")
    return y


def gdn_rmsnorm_gated(o, z, weight, eps: float = 1e-6, *, out=None):
    """o / rms(o) * weight * silu(z) over the last dimension d (64 or 128); o and z of the
    same shape and dtype, weight [d] fp32. Returns y (may be passed as o or z via `out`)."""
    lib = load_library()
    _need_cuda(o, z, weight, out)
    if o.shape != z.shape or o.dtype != z.dtype:
        raise ValueError("o and z must share shape and dtype")
    io = _io_dtype(o)
    d = o.shape[-1]
    y = out if out is not None else torch.empty_like(o)
    st = lib.gdn_rmsnorm_gated(_ptr(o), _ptr(z), io, _ptr(weight), float(eps), o.numel() // d, d,
                               _ptr(y), _stream(o.device))
    _check(st, "gdn_rmsnorm_gated")
    return y


def mixer_workspace_size(num_seqs, total_tokens, H_qk, H_v, d, io_dtype=torch.bfloat16) -> int:
    io = GDN_BF16 if io_dtype == torch.bfloat16 else GDN_FP32
    return int(load_library().gdn_mixer_prefill_workspace_size(num_seqs, total_tokens, H_qk,
                                                               H_v, d, d, io))


def gdn_mixer_prefill(x, conv_weight, conv_bias, cu_seqlens, a, b, A_log, dt_bias, z,
                      norm_weight, *, H_qk: int, conv_state_in=None, conv_state_out=None,
                      initial_state=None, eps: float = 1e-6, scale: float = 1.0,
                      output_final_state: bool = True, out=None, final_state=None,
                      workspace=None, impl: int = GDN_IMPL_AUTO,
                      timer: Optional[Timer] = None, fault: int = GDN_FAULT_NONE,
                      wait_limit_cycles: int = 0):
    """The mixer core in one call: y = RMSNorm(o) * w * SiLU(z) with o the gated delta
    rule over the causal conv1d + SiLU of x. Returns (y, final_state or None).

    x [T, (2 H_qk + H_v) d] (q | k | v channels, bf16 or fp32); conv_weight [C, K] fp32;
    conv_bias [C] fp32 or None; cu_seqlens int32 [N+1]; a, b [T, H_v] fp32; A_log, dt_bias
    [H_v] fp32; z [T, H_v, d] (x's dtype); norm_weight [d] fp32; conv_state_in /
    conv_state_out [N, K-1, C] or None (out may be in: updated in place); initial_state
    [N, H_v, d, d] fp32 or None.
    """
    lib = load_library()
    _need_cuda(x, conv_weight, conv_bias, cu_seqlens, a, b, A_log, dt_bias, z, norm_weight,
               conv_state_in, conv_state_out, initial_state, out, final_state, workspace)
    io = _io_dtype(x)
    T, C = x.shape
    _, H_v, d = z.shape
    K = conv_weight.shape[1]
    N = cu_seqlens.numel() - 1
    if C != (2 * H_qk + H_v) * d:
        raise ValueError("x must have (2 H_qk + H_v) d channels")
    y = out if out is not None else torch.empty_like(z)
    if output_final_state and final_state is None:
        final_state = torch.empty((N, H_v, d, d), device=x.device, dtype=torch.float32)
    if not output_final_state:
        final_state = None
    need = lib.gdn_mixer_prefill_workspace_size(N, T, H_qk, H_v, d, d, io)
    if workspace is None:
        workspace = torch.empty((max(int(need), 1),), device=x.device, dtype=torch.uint8)
    opts = _options(impl, fault, wait_limit_cycles, timer)
    st = lib.gdn_mixer_prefill(_ptr(x), io, _ptr(conv_weight), _ptr(conv_bias),
                               _ptr(conv_state_in), _ptr(conv_state_out), K, _ptr(a), _ptr(b),
                               _ptr(A_log), _ptr(dt_bias), _ptr(initial_state), _ptr(cu_seqlens),
                               N, T, H_qk, H_v, d, d, float(scale), _ptr(z), _ptr(norm_weight),
                               float(eps), _ptr(y), _ptr(final_state), _ptr(workspace),
                               workspace.numel(), opts, _stream(x.device))
    _check(st, "gdn_mixer_prefill")
    return y, final_state
