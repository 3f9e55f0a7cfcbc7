"""Pins for the fp64 oracle, checked against what the pages and mathematics fix.

No page prints a worked numeric example, so every pin is derived: brute force
in the spec matrix form, exact dyadic rationals, closed forms and
invariants, special cases that reduce to linear attention, structure
(packing, resume, head mapping) and the chunkwise identity of the
"Qwen3.5-MoE-35B-A3B architecture teardown", section 3.7. Each is chosen so that
a plausible slip in the oracle (the decay after the read instead of before, a
dropped beta, a transposed state, h % H_qk instead of h // r, a missing L2
norm, a wrong gate sign) fails at least one of them.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from tests.chunk_form import chunk_forward, l2n

rng = np.random.default_rng(1234)


def _rand(*shape):
    return rng.standard_normal(shape)


# ----------------------------------------------------------------- gates ----

def test_gates_closed_forms():
    # a + dt_bias = 0 -> softplus = ln 2, so g = -exp(A_log) ln 2.
    A_log = np.array([0.0, math.log(4.0), 1.7])
    dt = np.array([0.5, -0.25, 0.0])
    a = -dt[None, :].repeat(2, 0)
    b = np.array([[0.0, math.log(3.0), -math.log(3.0)], [50.0, -50.0, 0.0]])
    g, beta = oracle.gates(a, b, A_log, dt)
    assert np.allclose(g, -np.exp(A_log) * math.log(2.0), rtol=0, atol=1e-15)
    # sigmoid(0) = 1/2, sigmoid(ln 3) = 3/4, sigmoid(-ln 3) = 1/4
    assert beta[0].tolist() == pytest.approx([0.5, 0.75, 0.25], abs=1e-15)
    assert beta[1, 0] == pytest.approx(1.0, abs=1e-20)
    assert beta[1, 1] == pytest.approx(math.exp(-50.0), rel=1e-12)


def test_gates_sign_and_range():
    a, b = _rand(64, 8), _rand(64, 8)
    A_log = rng.uniform(0, math.log(16), 8)
    dt = rng.uniform(-1, 1, 8)
    g, beta = oracle.gates(a, b, A_log, dt)
    assert (g < 0).all() and (beta > 0).all() and (beta < 1).all()
    alpha = np.exp(g)
    assert (alpha > 0).all() and (alpha < 1).all()


def test_gates_match_library_softplus_sigmoid():
    # Special case that reduces to library routines (independent of the C code).
    a, b = _rand(128, 6) * 8, _rand(128, 6) * 8
    A_log = rng.uniform(0, math.log(16), 6)
    dt = rng.uniform(-1, 1, 6)
    g, beta = oracle.gates(a, b, A_log, dt)
    x = torch.from_numpy(a + dt)
    sp = torch.nn.functional.softplus(x, beta=1.0, threshold=1000.0).numpy()
    assert np.allclose(g, -np.exp(A_log) * sp, rtol=1e-14, atol=0)
    assert np.allclose(beta, torch.sigmoid(torch.from_numpy(b)).numpy(), rtol=1e-14, atol=0)


def test_gates_extremes():
    # alpha = 1 (a -> -inf), beta = 0 (b -> -inf), alpha = 0 (A_log large).
    a = np.array([[-1e30, 0.3]])
    b = np.array([[-1e30, 1e30]])
    g, beta = oracle.gates(a, b, np.array([0.0, 100.0]), np.array([0.0, 0.0]))
    assert g[0, 0] == 0.0 and np.exp(g[0, 0]) == 1.0
    assert np.exp(g[0, 1]) == 0.0
    assert beta[0, 0] == 0.0 and beta[0, 1] == 1.0
    assert np.isfinite(g[0, 0])


def test_chunk_cumsum_restarts():
    g = -rng.uniform(0, 1, (300, 3))
    cu = [0, 70, 70, 300]
    G = oracle.chunk_cumsum(g, cu, chunk=64)
    for s0, s1 in [(0, 70), (70, 300)]:
        for c0 in range(s0, s1, 64):
            c1 = min(c0 + 64, s1)
            assert np.allclose(G[c0:c1], np.cumsum(g[c0:c1], axis=0), atol=1e-14)


# ------------------------------------------- (a) brute force, matrix form ----

def _brute_force(q, k, v, g, beta, S0, H_qk, use_l2=True, scale=1.0):
    """S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T ; o_t = S_t q_t."""
    T, _, d_k = q.shape
    H_v, d_v = v.shape[1], v.shape[2]
    r = H_v // H_qk
    o = np.zeros((T, H_v, d_v))
    S_out = np.zeros((H_v, d_v, d_k))
    for h in range(H_v):
        S = S0[h].copy()
        for t in range(T):
            qt, kt = q[t, h // r], k[t, h // r]
            if use_l2:
                qt, kt = l2n(qt), l2n(kt)
            qt = qt * scale
            al, bt = math.exp(g[t, h]), beta[t, h]
            S = al * S @ (np.eye(d_k) - bt * np.outer(kt, kt)) + bt * np.outer(v[t, h], kt)
            o[t, h] = S @ qt
        S_out[h] = S
    return o, S_out


@pytest.mark.parametrize("T,H_qk,H_v,d_k,d_v", [(1, 1, 1, 2, 2), (3, 1, 2, 3, 2),
                                                 (4, 2, 4, 4, 3), (4, 1, 3, 2, 4)])
def test_brute_force_matrix_form(T, H_qk, H_v, d_k, d_v):
    q, k, v = _rand(T, H_qk, d_k), _rand(T, H_qk, d_k), _rand(T, H_v, d_v)
    g = -rng.uniform(0, 2, (T, H_v))
    beta = rng.uniform(0, 1, (T, H_v))
    S0 = _rand(H_v, d_v, d_k) * 0.3
    for scale in (1.0, 0.37):
        o, Sf = oracle.recurrent(q, k, v, g, beta, [0, T], S0[None], scale=scale)
        ob, Sb = _brute_force(q, k, v, g, beta, S0, H_qk, scale=scale)
        assert np.abs(o - ob).max() < 1e-12
        assert np.abs(Sf[0] - Sb).max() < 1e-12


def test_brute_force_exact_dyadic():
    """alpha = 1, dyadic q/k/v/beta, no L2 norm: every fp64 step is exact, so the
    oracle must equal the rational-arithmetic matrix form bit for bit."""
    T, d_k, d_v = 3, 3, 2
    vals = [Fraction(n, 4) for n in range(-6, 7)]
    rs = np.random.default_rng(7)
    pick = lambda *s: [[vals[i] for i in row] for row in rs.integers(0, len(vals), s)]
    Q, K, Vv = pick(T, d_k), pick(T, d_k), pick(T, d_v)
    B = [Fraction(1, 2), Fraction(3, 4), Fraction(1, 4)]
    S = [[Fraction(0)] * d_k for _ in range(d_v)]
    o_exact = []
    for t in range(T):
        # S (I - b k k^T) + b v k^T, with exact fractions
        kk = K[t]
        Sk = [sum(S[i][c] * kk[c] for c in range(d_k)) for i in range(d_v)]
        S = [[S[i][c] - B[t] * Sk[i] * kk[c] + B[t] * Vv[t][i] * kk[c] for c in range(d_k)]
             for i in range(d_v)]
        o_exact.append([sum(S[i][c] * Q[t][c] for c in range(d_k)) for i in range(d_v)])
    f = lambda M: np.array([[float(x) for x in row] for row in M])
    q = f(Q)[:, None, :]
    k = f(K)[:, None, :]
    v = f(Vv)[:, None, :]
    g = np.zeros((T, 1))
    beta = np.array([[float(x)] for x in B])
    o, Sf = oracle.recurrent(q, k, v, g, beta, [0, T], use_l2norm=False)
    assert (o[:, 0, :] == f(o_exact)).all()
    assert (Sf[0, 0] == f(S)).all()


# ------------------------------------------- (b) exact write with beta=1 ----

def test_beta_one_unit_key_stores_value():
    """beta = 1 and |k| = 1 give S_t k_t = v_t after the write; with q_t = k_t the
    read-out returns v_t exactly, for any decay and any prior state."""
    T, d_k, d_v = 20, 8, 5
    k = l2n(_rand(T, 1, d_k), eps=0.0)
    v = _rand(T, 1, d_v)
    g = -rng.uniform(0, 1, (T, 1))
    S0 = _rand(1, 1, d_v, d_k)
    o, _ = oracle.recurrent(k, k, v, g, np.ones((T, 1)), [0, T], S0, use_l2norm=False)
    assert np.abs(o - v).max() < 1e-12


# ------------------------------------------------ (c) alpha/beta limits ----

def test_identity_gates_leave_state():
    """alpha = 1, beta = 0: S never changes and o_t = S0 q_t."""
    T, H_qk, H_v, d = 17, 2, 4, 6
    q, k, v = _rand(T, H_qk, d), _rand(T, H_qk, d), _rand(T, H_v, d)
    S0 = _rand(1, H_v, d, d)
    o, Sf = oracle.recurrent(q, k, v, np.zeros((T, H_v)), np.zeros((T, H_v)), [0, T], S0)
    assert np.array_equal(Sf, S0)
    qn = l2n(q)
    for h in range(H_v):
        assert np.abs(o[:, h] - qn[:, h // 2] @ S0[0, h].T).max() < 1e-13


def test_zero_alpha_resets_state():
    """alpha = 0: S_t = beta_t v_t k_t^T, o_t = beta_t v_t (k_t . q_t)."""
    T, d_k, d_v = 9, 4, 3
    q, k, v = _rand(T, 1, d_k), _rand(T, 1, d_k), _rand(T, 1, d_v)
    beta = rng.uniform(0.1, 1, (T, 1))
    S0 = _rand(1, 1, d_v, d_k)
    o, Sf = oracle.recurrent(q, k, v, np.full((T, 1), -np.inf), beta, [0, T], S0)
    qn, kn = l2n(q[:, 0]), l2n(k[:, 0])
    expect = beta * v[:, 0] * (kn * qn).sum(-1, keepdims=True)
    assert np.abs(o[:, 0] - expect).max() < 1e-13
    assert np.abs(Sf[0, 0] - beta[-1, 0] * np.outer(v[-1, 0], kn[-1])).max() < 1e-13


# -------------------------------- (d) orthogonal keys = linear attention ----

@pytest.mark.parametrize("gated", [False, True])
def test_orthogonal_keys_reduce_to_linear_attention(gated):
    """With mutually orthogonal keys and S0 = 0 the delta term S_{t-1} k_t
    vanishes, so the rule is (gated) linear attention:
    o_t = sum_{j<=t} (prod_{j<s<=t} alpha_s) beta_j v_j k_j^T q_t."""
    d_k, d_v, T = 8, 5, 8
    Qm, _ = np.linalg.qr(_rand(d_k, d_k))
    k = (Qm.T * rng.uniform(0.5, 2, (d_k, 1)))[:, None, :]  # orthogonal rows
    q, v = _rand(T, 1, d_k), _rand(T, 1, d_v)
    beta = rng.uniform(0.2, 1, (T, 1))
    g = -rng.uniform(0, 1, (T, 1)) if gated else np.zeros((T, 1))
    o, _ = oracle.recurrent(q, k, v, g, beta, [0, T])
    qn, kn = l2n(q[:, 0]), l2n(k[:, 0])
    for t in range(T):
        acc = np.zeros(d_v)
        for j in range(t + 1):
            decay = math.exp(g[j + 1:t + 1, 0].sum())
            acc += decay * beta[j, 0] * v[j, 0] * (kn[j] @ qn[t])
        assert np.abs(o[t, 0] - acc).max() < 1e-12


# -------------------------- (e) orthonormal keys: perfect associative recall ----

def test_orthonormal_keys_recall():
    d_k, d_v, T = 6, 4, 6
    Qm, _ = np.linalg.qr(_rand(d_k, d_k))
    k = Qm.T[:, None, :]
    v = _rand(T, 1, d_v)
    q = _rand(T, 1, d_k)
    _, Sf = oracle.recurrent(q, k, v, np.zeros((T, 1)), np.ones((T, 1)), [0, T],
                             use_l2norm=False)
    for j in range(T):
        assert np.abs(Sf[0, 0] @ k[j, 0] - v[j, 0]).max() < 1e-12


# ------------------------------------------------ (f) affine linearity ----

def test_joint_linearity_in_state_and_values():
    T, H_qk, H_v, d = 40, 1, 2, 8
    q, k = _rand(T, H_qk, d), _rand(T, H_qk, d)
    g = -rng.uniform(0, 1, (T, H_v))
    beta = rng.uniform(0, 1, (T, H_v))
    Va, Vb = _rand(T, H_v, d), _rand(T, H_v, d)
    Sa, Sb = _rand(1, H_v, d, d), _rand(1, H_v, d, d)
    c1, c2 = 0.7, -1.3
    oa, Fa = oracle.recurrent(q, k, Va, g, beta, [0, T], Sa)
    ob, Fb = oracle.recurrent(q, k, Vb, g, beta, [0, T], Sb)
    oc, Fc = oracle.recurrent(q, k, c1 * Va + c2 * Vb, g, beta, [0, T], c1 * Sa + c2 * Sb)
    assert np.abs(oc - (c1 * oa + c2 * ob)).max() < 1e-12
    assert np.abs(Fc - (c1 * Fa + c2 * Fb)).max() < 1e-12


# ------------------------------------------------------- (g) structure ----

def _rand_problem(lens, H_qk=2, H_v=4, d_k=8, d_v=6, with_state=True):
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return dict(q=_rand(T, H_qk, d_k), k=_rand(T, H_qk, d_k), v=_rand(T, H_v, d_v),
                a=_rand(T, H_v), b=_rand(T, H_v),
                A_log=rng.uniform(0, math.log(16), H_v), dt_bias=rng.uniform(-1, 1, H_v),
                cu=cu, S0=_rand(len(lens), H_v, d_v, d_k) * 0.1 if with_state else None)


def test_packed_equals_separate_runs():
    lens = [5, 1, 13, 7]
    P = _rand_problem(lens)
    o, Sf = oracle.forward(P["q"], P["k"], P["v"], P["a"], P["b"], P["A_log"], P["dt_bias"],
                           P["cu"], P["S0"])
    cu = P["cu"]
    for n in range(len(lens)):
        s = slice(cu[n], cu[n + 1])
        on, Sn = oracle.forward(P["q"][s], P["k"][s], P["v"][s], P["a"][s], P["b"][s],
                                P["A_log"], P["dt_bias"], [0, lens[n]], P["S0"][n:n + 1])
        assert np.array_equal(o[s], on) and np.array_equal(Sf[n], Sn[0])


def test_split_resume_equals_single_pass():
    P = _rand_problem([30])
    args = lambda s: (P["q"][s], P["k"][s], P["v"][s], P["a"][s], P["b"][s], P["A_log"],
                      P["dt_bias"])
    o, Sf = oracle.forward(*args(slice(0, 30)), [0, 30], P["S0"])
    o1, S1 = oracle.forward(*args(slice(0, 11)), [0, 11], P["S0"])
    o2, S2 = oracle.forward(*args(slice(11, 30)), [0, 19], S1)
    assert np.array_equal(np.concatenate([o1, o2]), o) and np.array_equal(S2, Sf)


def test_decode_steps_equal_prefill():
    P = _rand_problem([12], with_state=True)
    o, Sf = oracle.forward(P["q"], P["k"], P["v"], P["a"], P["b"], P["A_log"], P["dt_bias"],
                           P["cu"], P["S0"])
    S = P["S0"]
    for t in range(12):
        s = slice(t, t + 1)
        ot, S = oracle.decode_step(P["q"][s], P["k"][s], P["v"][s], P["a"][s], P["b"][s],
                                   P["A_log"], P["dt_bias"], S)
        assert np.array_equal(ot[0], o[t])
    assert np.array_equal(S, Sf)


def test_head_mapping_is_repeat_interleave():
    """V head h reads QK head h // (H_v / H_qk) (repeat_interleave on dim 2)."""
    P = _rand_problem([9], H_qk=2, H_v=6, with_state=False)
    o, _ = oracle.forward(P["q"], P["k"], P["v"], P["a"], P["b"], P["A_log"], P["dt_bias"],
                          P["cu"])
    for h in range(6):
        j = h // 3
        oh, _ = oracle.forward(P["q"][:, j:j + 1], P["k"][:, j:j + 1], P["v"][:, h:h + 1],
                               P["a"][:, h:h + 1], P["b"][:, h:h + 1], P["A_log"][h:h + 1],
                               P["dt_bias"][h:h + 1], P["cu"])
        assert np.array_equal(o[:, h], oh[:, 0])


def test_l2norm_makes_qk_scale_free():
    P = _rand_problem([10], with_state=False)
    o, Sf = oracle.forward(P["q"], P["k"], P["v"], P["a"], P["b"], P["A_log"], P["dt_bias"],
                           P["cu"])
    o2, Sf2 = oracle.forward(P["q"] * 3.0, P["k"] * 2.0, P["v"], P["a"], P["b"], P["A_log"],
                             P["dt_bias"], P["cu"])
    # equal up to the 1e-6 epsilon inside the norm (|k|^2 is about 8 here)
    assert np.abs(o - o2).max() < 1e-6 and np.abs(Sf - Sf2).max() < 1e-6
    o3, _ = oracle.forward(P["q"] * 3.0, P["k"] * 2.0, P["v"], P["a"], P["b"], P["A_log"],
                           P["dt_bias"], P["cu"], use_l2norm=False)
    assert np.abs(o - o3).max() > 1e-2  # the norm is really applied


def test_single_token_closed_form():
    """From a zero state one token gives S = beta v k^T and o = beta v (k . q)."""
    q, k, v = _rand(1, 1, 5), _rand(1, 1, 5), _rand(1, 1, 3)
    g, beta = np.array([[-0.4]]), np.array([[0.3]])
    o, Sf = oracle.recurrent(q, k, v, g, beta, [0, 1])
    qn, kn = l2n(q[0, 0]), l2n(k[0, 0])
    assert np.abs(o[0, 0] - 0.3 * v[0, 0] * (kn @ qn)).max() < 1e-14
    assert np.abs(Sf[0, 0] - 0.3 * np.outer(v[0, 0], kn)).max() < 1e-14


# ------------------------------------------- (h) chunkwise identity ----

@pytest.mark.parametrize("lens", [[1], [63], [64], [65], [127, 64, 3, 200]])
def test_chunk_identity_matches_recurrence(lens):
    P = _rand_problem(lens, H_qk=1, H_v=2, d_k=16, d_v=8)
    g, beta = oracle.gates(P["a"], P["b"], P["A_log"], P["dt_bias"])
    o, Sf = oracle.recurrent(P["q"], P["k"], P["v"], g, beta, P["cu"], P["S0"])
    oc, Sc = chunk_forward(P["q"], P["k"], P["v"], g, beta, P["cu"], P["S0"])
    scale_o = np.abs(o).max()
    assert np.abs(o - oc).max() < 1e-10 * max(1.0, scale_o)
    assert np.abs(Sf - Sc).max() < 1e-10 * max(1.0, np.abs(Sf).max())


def test_chunk_identity_slow_decay():
    """A_log = -4 (alpha near 0.98) keeps long-range carry alive across chunks."""
    P = _rand_problem([200], H_qk=1, H_v=1, d_k=16, d_v=16)
    g, beta = oracle.gates(P["a"], P["b"], np.array([-4.0]), P["dt_bias"][:1])
    o, Sf = oracle.recurrent(P["q"], P["k"], P["v"][:, :1], g, beta, P["cu"], P["S0"][:, :1])
    oc, Sc = chunk_forward(P["q"], P["k"], P["v"][:, :1], g, beta, P["cu"], P["S0"][:, :1])
    assert np.abs(o - oc).max() < 1e-10 * np.abs(o).max()
    assert np.abs(Sf - Sc).max() < 1e-10 * np.abs(Sf).max()
