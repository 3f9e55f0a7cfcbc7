"""The state map of a stretch of tokens is affine, in fp64 on the CPU (the oracle).

For any run of tokens of one (sequence, V head), the gated delta rule takes the state before
it to the state after it as S_end = S_start M + B ("Qwen3.5-MoE-35B-A3B architecture
teardown", section 3.3, the recurrence; section 3.7, the chunk form's state update), where
M (d_k x d_k) is what the run does to S_start = I with v = 0 and B (d_v x d_k) what it does to
S_start = 0 with the real v. The outputs split the same way. This is what a prefill that
splits one sequence along T relies on: each segment's (M, B) computed in parallel, a short
sequential combine, then each segment's outputs from its true starting state.
"""
import numpy as np

import oracle

D = 16  # d_k = d_v, so that S_start = I is a state of the same shape


def _inputs(T, H_qk, H_v, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H_qk, D))
    k = rng.standard_normal((T, H_qk, D))
    v = rng.standard_normal((T, H_v, D))
    g = -np.log1p(np.exp(rng.standard_normal((T, H_v)))) * 0.3
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H_v))))
    return q, k, v, g, beta


def _run(q, k, v, g, beta, S0):
    return oracle.recurrent(q, k, v, g, beta, np.array([0, v.shape[0]]), S0[None])


def _map(q, k, v, g, beta):
    """(M, B) of a run, per V head: M from S0 = I and v = 0, B from S0 = 0."""
    H_v = v.shape[1]
    eye = np.broadcast_to(np.eye(D), (H_v, D, D)).copy()
    _, M = _run(q, k, np.zeros_like(v), g, beta, eye)
    _, B = _run(q, k, v, g, beta, np.zeros((H_v, D, D)))
    return M[0], B[0]


def test_one_token_map_is_the_closed_form():
    """One token: M = alpha (I - beta k^ k^T) and B = beta v k^T (from the recurrence
    written out, not from the oracle's code)."""
    q, k, v, g, beta = _inputs(1, 1, 2, seed=11)
    M, B = _map(q, k, v, g, beta)
    kh = k[0, 0] / np.sqrt(np.sum(k[0, 0] ** 2) + 1e-6)
    for h in range(2):
        alpha = np.exp(g[0, h])
        assert np.allclose(M[h], alpha * (np.eye(D) - beta[0, h] * np.outer(kh, kh)),
                           rtol=1e-12, atol=1e-14)
        assert np.allclose(B[h], beta[0, h] * np.outer(v[0, h], kh), rtol=1e-12, atol=1e-14)


def test_final_state_is_affine_in_the_initial_state():
    q, k, v, g, beta = _inputs(200, 1, 2, seed=12)
    M, B = _map(q, k, v, g, beta)
    X = np.random.default_rng(13).standard_normal((2, D, D))
    _, S = _run(q, k, v, g, beta, X)
    for h in range(2):
        ref = S[0, h]
        assert np.abs(X[h] @ M[h] + B[h] - ref).max() <= 1e-10 * np.abs(ref).max()


def test_outputs_split_into_state_part_and_input_part():
    q, k, v, g, beta = _inputs(150, 1, 2, seed=14)
    X = np.random.default_rng(15).standard_normal((2, D, D))
    o, _ = _run(q, k, v, g, beta, X)
    o_state, _ = _run(q, k, np.zeros_like(v), g, beta, X)
    o_input, _ = _run(q, k, v, g, beta, np.zeros((2, D, D)))
    assert np.abs(o_state + o_input - o).max() <= 1e-10 * np.abs(o).max()


def test_split_along_t_equals_one_run():
    """Segments [0, 64), [64, 150), [150, 257): per-segment maps, a sequential combine of the
    starting states, then each segment from its true start; outputs and final state equal one
    run over all tokens. The QK heads are shared by two V heads each."""
    q, k, v, g, beta = _inputs(257, 2, 4, seed=16)
    S0 = np.random.default_rng(17).standard_normal((4, D, D)) * 0.1
    o_ref, S_ref = _run(q, k, v, g, beta, S0)
    bounds = [0, 64, 150, 257]
    segs = [slice(a, b) for a, b in zip(bounds[:-1], bounds[1:])]
    maps = [_map(q[s], k[s], v[s], g[s], beta[s]) for s in segs]  # independent of each other
    starts = [S0]
    for M, B in maps[:-1]:
        starts.append(np.einsum("hij,hjk->hik", starts[-1], M) + B)
    o = np.concatenate([_run(q[s], k[s], v[s], g[s], beta[s], st)[0]
                        for s, st in zip(segs, starts)])
    M, B = maps[-1]
    S_end = np.einsum("hij,hjk->hik", starts[-1], M) + B
    assert np.abs(o - o_ref).max() <= 1e-10 * np.abs(o_ref).max()
    assert np.abs(S_end - S_ref[0]).max() <= 1e-10 * np.abs(S_ref).max()
