"""The cross-chunk identity behind the Gram-matrix prefill schedule, in fp64 on the CPU.

With S_c the state before chunk c, gamma_c = e^{G_last} of chunk c and the chunk's state
increment U_c = Vnew_c^T diag(e^{G_last - G}) K_c (the chunkwise form of the gated delta
rule, "Qwen3.5-MoE-35B-A3B architecture teardown", section 3.7, steps 3-6):

    S_{c+1} K_{c+1}^T = gamma_c S_c K_{c+1}^T + (Vnew_c^T diag(e^{G_last - G})) (K_c K_{c+1}^T)

so the product the next chunk needs first can be formed from the previous chunk's state and
the key Gram matrix K_c K_{c+1}^T, which does not depend on the state. The chunk loop below
is the one of tests/chunk_form.py, recording every chunk's quantities.
"""
import numpy as np

from tests.chunk_form import chunk_forward, l2n


def _chunks(q, k, v, g, beta, chunk=64):
    T, _, d_k = k.shape
    d_v = v.shape[2]
    S = np.zeros((d_v, d_k))
    out = []
    for cs in range(0, T, chunk):
        ce = min(cs + chunk, T)
        K = l2n(k[cs:ce, 0])
        V = v[cs:ce, 0]
        G = np.cumsum(g[cs:ce, 0])
        bt = beta[cs:ce, 0]
        L = ce - cs
        diff = G[:, None] - G[None, :]
        incl = np.tril(np.ones((L, L), dtype=bool))
        Gam = np.where(incl, np.exp(np.where(incl, diff, 0.0)), 0.0)
        A = np.tril(bt[:, None] * Gam * (K @ K.T), -1)
        Tm = np.linalg.inv(np.eye(L) + A)
        Vn = Tm @ (bt[:, None] * V) - (Tm @ ((bt * np.exp(G))[:, None] * K)) @ S.T
        Wt = Vn.T * np.exp(G[-1] - G)[None, :]          # decay-scaled Vnew^T, d_v x L
        out.append(dict(S=S.copy(), K=K, gamma=np.exp(G[-1]), Wt=Wt))
        S = np.exp(G[-1]) * S + Wt @ K
    return out, S


def _inputs(T, seed, a_log=0.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, 1, 32))
    k = rng.standard_normal((T, 1, 32))
    v = rng.standard_normal((T, 1, 16))
    g = -np.exp(a_log) * np.log1p(np.exp(rng.standard_normal((T, 1))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, 1))))
    return q, k, v, g, beta


def test_state_k_product_from_previous_chunk_and_gram():
    q, k, v, g, beta = _inputs(64 * 5 + 17, seed=3, a_log=-2.0)
    ch, _ = _chunks(q, k, v, g, beta)
    for c in range(len(ch) - 1):
        a, b = ch[c], ch[c + 1]
        direct = b["S"] @ b["K"].T
        gram = a["K"] @ b["K"].T                          # K_c K_{c+1}^T
        via = a["gamma"] * (a["S"] @ b["K"].T) + a["Wt"] @ gram
        assert np.allclose(via, direct, rtol=1e-10, atol=1e-12)


def test_recorded_loop_matches_chunk_form():
    """The loop above is the chunk form's own (same final state), so the identity is checked
    on the quantities the prefill actually propagates."""
    q, k, v, g, beta = _inputs(200, seed=5)
    _, S = _chunks(q, k, v, g, beta)
    _, Sf = chunk_forward(q, k, v, g, beta, np.array([0, 200]))
    assert np.allclose(S, Sf[0, 0], rtol=1e-12, atol=1e-12)


def test_gram_term_vanishes_without_increment():
    """beta = 0 everywhere: no writes, so the state only decays and the Gram term is zero."""
    q, k, v, g, beta = _inputs(130, seed=7)
    beta[:] = 0.0
    ch, _ = _chunks(q, k, v, g, beta)
    for c in range(len(ch)):
        assert np.abs(ch[c]["Wt"]).max() == 0.0
