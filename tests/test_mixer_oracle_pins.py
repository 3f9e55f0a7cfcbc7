"""Pins for the oracle of the steps around the delta rule: the causal depthwise
convolution + SiLU ("Qwen3.5-MoE-35B-A3B architecture teardown", 3.3 phase 2) and the
gated RMSNorm (3.3 phase 4). Each pin checks the oracle against something other than
its own formula: a library routine (scipy's FIR filter, torch's rms_norm and silu),
closed forms, or structure (chaining the conv cache, packing sequences).
"""
import numpy as np
import pytest
import torch
from scipy.signal import lfilter

import oracle

RNG = np.random.default_rng(1234)


def _silu(x):
    return x / (1.0 + np.exp(-x))


# ----------------------------------------------------------------- conv1d + SiLU --

def test_conv_matches_fir_filter():
    """Per channel the convolution is an FIR filter of the cache-prefixed input with
    taps reversed (the last tap multiplies the current token)."""
    T, C, K = 37, 6, 4
    x = RNG.standard_normal((T, C))
    w = RNG.standard_normal((C, K))
    b = RNG.standard_normal(C)
    st = RNG.standard_normal((1, K - 1, C))
    y, so = oracle.conv1d_silu(x, w, b, [0, T], state_in=st)
    for c in range(C):
        xs = np.concatenate([st[0, :, c], x[:, c]])
        ref = lfilter(w[c, ::-1], [1.0], xs)[K - 1:] + b[c]
        np.testing.assert_allclose(y[:, c], _silu(ref), rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(so[0], x[T - (K - 1):])


def test_conv_identity_tap_is_plain_silu():
    T, C, K = 20, 3, 4
    x = RNG.standard_normal((T, C))
    w = np.zeros((C, K))
    w[:, K - 1] = 1.0
    y, _ = oracle.conv1d_silu(x, w, None, [0, 7, T])
    np.testing.assert_allclose(y, _silu(x), rtol=1e-14)


def test_conv_zero_cache_is_causal_zero_padding():
    """Without a cache, the first K-1 outputs see zeros before the sequence: a single
    unit input at a sequence's first token yields the taps, in order, at t = 0..K-1."""
    C, K = 2, 4
    x = np.zeros((8, C))
    x[0] = 1.0
    w = RNG.standard_normal((C, K))
    y, _ = oracle.conv1d_silu(x, w, None, [0, 8])
    for t in range(K):
        np.testing.assert_allclose(y[t], _silu(w[:, K - 1 - t]), rtol=1e-14)
    np.testing.assert_allclose(y[K:], _silu(np.zeros((8 - K, C))), atol=0)


def test_conv_cache_chaining_equals_one_pass():
    """prefill(T1) then prefill(T2) from its cache == prefill(T1 + T2): the conv cache
    hand-off the pages describe for prefill -> decode."""
    T, C, K = 50, 5, 4
    x = RNG.standard_normal((T, C))
    w = RNG.standard_normal((C, K))
    b = RNG.standard_normal(C)
    y, so = oracle.conv1d_silu(x, w, b, [0, T])
    for split in (1, 2, 3, 17):
        y1, s1 = oracle.conv1d_silu(x[:split], w, b, [0, split])
        y2, s2 = oracle.conv1d_silu(x[split:], w, b, [0, T - split], state_in=s1)
        np.testing.assert_allclose(np.concatenate([y1, y2]), y, rtol=1e-14)
        np.testing.assert_array_equal(s2, so)


def test_conv_token_by_token_decode_equals_prefill():
    T, C, K = 9, 4, 4
    x = RNG.standard_normal((T, C))
    w = RNG.standard_normal((C, K))
    y, so = oracle.conv1d_silu(x, w, None, [0, T])
    st = np.zeros((1, K - 1, C))
    for t in range(T):
        yt, st = oracle.conv1d_silu(x[t:t + 1], w, None, [0, 1], state_in=st)
        np.testing.assert_allclose(yt[0], y[t], rtol=1e-14)
    np.testing.assert_array_equal(st, so)


def test_conv_packing_and_short_sequences():
    """Packed sequences (including empty and shorter-than-cache ones) equal separate calls;
    a short sequence's cache keeps the older cached positions."""
    C, K = 3, 4
    lens = [5, 0, 1, 2, 9]
    cu = np.concatenate([[0], np.cumsum(lens)])
    x = RNG.standard_normal((cu[-1], C))
    w = RNG.standard_normal((C, K))
    st = RNG.standard_normal((len(lens), K - 1, C))
    y, so = oracle.conv1d_silu(x, w, None, cu, state_in=st)
    for n, L in enumerate(lens):
        yn, sn = oracle.conv1d_silu(x[cu[n]:cu[n + 1]], w, None, [0, L], state_in=st[n:n + 1])
        np.testing.assert_allclose(y[cu[n]:cu[n + 1]], yn, rtol=1e-14)
        np.testing.assert_array_equal(so[n], sn[0])
    np.testing.assert_array_equal(so[1], st[1])                       # empty: unchanged
    np.testing.assert_array_equal(so[2], np.concatenate([st[2, 1:], x[cu[2]:cu[3]]]))  # len 1
    np.testing.assert_array_equal(so[3], np.concatenate([st[3, 2:], x[cu[3]:cu[4]]]))  # len 2


# ----------------------------------------------------------------- gated RMSNorm --

def test_rmsnorm_gated_matches_torch():
    o = RNG.standard_normal((17, 128))
    z = RNG.standard_normal((17, 128))
    w = RNG.standard_normal(128)
    y = oracle.rmsnorm_gated(o, z, w, eps=1e-6)
    ot, zt, wt = (torch.tensor(a, dtype=torch.float64) for a in (o, z, w))
    ref = torch.nn.functional.rms_norm(ot, (128,), wt, eps=1e-6) * torch.nn.functional.silu(zt)
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-12, atol=1e-14)


def test_rmsnorm_gated_closed_forms():
    d = 64
    w = RNG.standard_normal(d)
    z = RNG.standard_normal((3, d))
    c = np.array([[2.5], [-0.75], [1e-4]])
    o = np.repeat(c, d, axis=1)                     # constant rows: |o| / rms = 1 up to eps
    y = oracle.rmsnorm_gated(o, z, w, eps=1e-6)
    expect = np.sign(c) / np.sqrt(1.0 + 1e-6 / c ** 2) * w * _silu(z)
    np.testing.assert_allclose(y, expect, rtol=1e-12)
    # scale invariance (eps aside) and a zero gate
    o2 = RNG.standard_normal((4, d))
    z2 = RNG.standard_normal((4, d))
    np.testing.assert_allclose(oracle.rmsnorm_gated(1e3 * o2, z2, w, eps=0.0),
                               oracle.rmsnorm_gated(o2, z2, w, eps=0.0), rtol=1e-12)
    assert np.all(oracle.rmsnorm_gated(o2, np.zeros_like(z2), w) == 0.0)
