"""Gated DeltaNet oracle: a plain sequential fp64 CPU reference.

TEST INFRASTRUCTURE ONLY. The test suite, the package's smoke check and the
benchmark's CPU-baseline leg are the only callers. The CUDA product path shares
no code with this package and never imports it.

The arithmetic lives in ``gdn_oracle.c`` (plain C, fp64, OpenMP over the
independent (sequence, V head) units). This module only builds that file,
loads it and marshals numpy arrays to it. Every input is converted to float64
exactly (bf16 values are upcast without rounding), so the oracle sees the same
numbers the GPU path sees.

Functions and the passages they follow:
  gates            -- beta = sigmoid(b); g = -exp(A_log) * softplus(a + dt_bias)
                      ("Qwen3.5 observation notes", "Qwen3_5MoeGatedDeltaNet")
  chunk_cumsum     -- cumulative sum of g inside each 64-token chunk
                      ("Qwen3.5-MoE-35B-A3B architecture teardown", 3.7 step 3)
  recurrent        -- the gated delta rule token by token, given g and beta
  forward          -- gates followed by the recurrence
  decode_step      -- one token per sequence from a stored state (the same
                      recurrence with a length-1 sequence per slot)
  conv1d_silu      -- causal depthwise convolution + SiLU over the q/k/v channels,
                      with the per-sequence conv cache in and out (``mixer_oracle.c``;
                      "Qwen3.5-MoE-35B-A3B architecture teardown", 3.3 phase 2)
  rmsnorm_gated    -- RMSNorm(o) * w * SiLU(z) per row (3.3 phase 4)
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_SRCS = [_SRC, os.path.join(_HERE, "mixer_oracle.c")]
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

CHUNK = 64


def build(force: bool = False) -> str:
    """Compile the oracle's C sources into liboracle.so next to them (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or any(
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(src) for src in _SRCS
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", *_SRCS, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.oracle_gates.argtypes = [P, P, P, P, i64, i32, P, P]
        lib.oracle_chunk_cumsum.argtypes = [P, P, i32, i32, i32, P]
        lib.oracle_gdn_recurrent.argtypes = [
            P, P, P, P, P, P, P, i32, i32, i32, i32, i32, f64, i32, P, P
        ]
        lib.oracle_gdn_forward.argtypes = [
            P, P, P, P, P, P, P, P, P, i32, i64, i32, i32, i32, i32, f64, i32, P, P
        ]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_conv1d_silu.argtypes = [P, P, P, P, P, i32, i32, i32, P, P]
        lib.oracle_rmsnorm_gated.argtypes = [P, P, P, f64, i64, i32, P]
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact upcast to a C-contiguous float64 array (accepts numpy or torch)."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: upcast through float32 is exact for bf16
        x = x.detach().cpu().float().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    """OpenMP threads the oracle's parallel regions use."""
    return int(_load().oracle_num_threads())


def gates(a, b, A_log, dt_bias):
    """Return (g, beta), each shaped like a ([T, H_v])."""
    lib = _load()
    a, b, A_log, dt_bias = _f64(a), _f64(b), _f64(A_log), _f64(dt_bias)
    T, H_v = a.shape
    g = np.empty_like(a)
    beta = np.empty_like(a)
    lib.oracle_gates(_ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias), T, H_v,
                     _ptr(g), _ptr(beta))
    return g, beta


def chunk_cumsum(g, cu_seqlens, chunk: int = CHUNK):
    """Inclusive cumsum of g ([T, H_v]) restarting every `chunk` tokens of each sequence."""
    lib = _load()
    g = _f64(g)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    G = np.empty_like(g)
    lib.oracle_chunk_cumsum(_ptr(g), _ptr(cu), len(cu) - 1, g.shape[1], chunk, _ptr(G))
    return G


def _shapes(q, v, cu):
    T, H_qk, d_k = q.shape
    T2, H_v, d_v = v.shape
    assert T == T2 and H_v % H_qk == 0 and cu[0] == 0 and cu[-1] == T
    return T, H_qk, H_v, d_k, d_v


def recurrent(q, k, v, g, beta, cu_seqlens, initial_state=None, scale: float = 1.0,
              use_l2norm: bool = True, want_final: bool = True):
    """The gated delta rule given g and beta. Returns (o, final_state or None).

    q, k [T, H_qk, d_k]; v [T, H_v, d_v]; g, beta [T, H_v];
    initial_state [N, H_v, d_v, d_k] (value-major, o = S q) or None for zeros.
    """
    lib = _load()
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    T, H_qk, H_v, d_k, d_v = _shapes(q, v, cu)
    N = len(cu) - 1
    S0 = _f64(initial_state)
    o = np.empty((T, H_v, d_v))
    Sf = np.empty((N, H_v, d_v, d_k)) if want_final else None
    lib.oracle_gdn_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                             _ptr(cu), N, H_qk, H_v, d_k, d_v, float(scale),
                             int(bool(use_l2norm)), _ptr(o), _ptr(Sf))
    return o, Sf


def forward(q, k, v, a, b, A_log, dt_bias, cu_seqlens, initial_state=None,
            scale: float = 1.0, use_l2norm: bool = True, want_final: bool = True):
    """Gates from (a, b, A_log, dt_bias), then the recurrence. Returns (o, final_state)."""
    lib = _load()
    q, k, v, a, b, A_log, dt_bias = map(_f64, (q, k, v, a, b, A_log, dt_bias))
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    T, H_qk, H_v, d_k, d_v = _shapes(q, v, cu)
    N = len(cu) - 1
    S0 = _f64(initial_state)
    o = np.empty((T, H_v, d_v))
    Sf = np.empty((N, H_v, d_v, d_k)) if want_final else None
    lib.oracle_gdn_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(A_log),
                           _ptr(dt_bias), _ptr(S0), _ptr(cu), N, T, H_qk, H_v, d_k, d_v,
                           float(scale), int(bool(use_l2norm)), _ptr(o), _ptr(Sf))
    return o, Sf


def decode_step(q, k, v, a, b, A_log, dt_bias, state, scale: float = 1.0):
    """One token for each of N sequences from state [N, H_v, d_v, d_k].

    q, k [N, H_qk, d_k]; v [N, H_v, d_v]; a, b [N, H_v]. Returns (o [N, H_v, d_v],
    new_state). The input state is not modified.
    """
    N = _f64(q).shape[0]
    cu = np.arange(N + 1, dtype=np.int64)
    return forward(q, k, v, a, b, A_log, dt_bias, cu, initial_state=state, scale=scale)


def conv1d_silu(x, weight, bias, cu_seqlens, state_in=None, want_state: bool = True):
    """Causal depthwise convolution + SiLU. Returns (y [T, C], state_out [N, K-1, C] or None).

    x [T, C]; weight [C, K] (weight[:, K-1] multiplies the current token); bias [C] or
    None; state_in [N, K-1, C] (the K-1 positions before each sequence, oldest first) or
    None for zeros.
    """
    lib = _load()
    x, w, bias, state_in = _f64(x), _f64(weight), _f64(bias), _f64(state_in)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    T, C = x.shape
    K = w.shape[1]
    N = len(cu) - 1
    assert w.shape[0] == C and cu[0] == 0 and cu[-1] == T
    y = np.empty_like(x)
    so = np.empty((N, K - 1, C)) if want_state else None
    lib.oracle_conv1d_silu(_ptr(x), _ptr(w), _ptr(bias), _ptr(state_in), _ptr(cu), N, C, K,
                           _ptr(y), _ptr(so))
    return y, so


def rmsnorm_gated(o, z, weight, eps: float = 1e-6):
    """y = o / sqrt(mean(o^2) + eps) * weight * silu(z) over the last axis (length d)."""
    lib = _load()
    o, z, w = _f64(o), _f64(z), _f64(weight)
    d = o.shape[-1]
    rows = o.size // d
    y = np.empty_like(o)
    lib.oracle_rmsnorm_gated(_ptr(o), _ptr(z), _ptr(w), float(eps), rows, d, _ptr(y))
    return y
