"""The chunkwise form of the gated delta rule, in plain numpy fp64.

Test helper only: it checks, on the CPU, the algebra that the CUDA prefill
kernel implements ("Qwen3.5-MoE-35B-A3B architecture teardown", section 3.7,
steps 3-6: the in-chunk decay mask, the triangular correction, the inter-chunk
scan and the per-chunk state update), restated from the recurrence:

  G_i  = sum_{s<=i} g_s inside the chunk,  Gamma_ij = exp(G_i - G_j) (i >= j)
  A    = strictly-lower(beta_i Gamma_ij k_i . k_j)
  T    = (I + A)^-1
  U    = T diag(beta) V,     W = T diag(beta e^G) K
  Vnew = U - W S0^T
  O    = diag(e^G) Q S0^T + (Q K^T (.) Gamma_incl) Vnew
  S    = e^{G_last} S0 + Vnew^T diag(e^{G_last - G}) K
with S value-major (d_v x d_k).
"""
import numpy as np


def l2n(x, eps=1e-6):
    return x / np.sqrt((x * x).sum(-1, keepdims=True) + eps)


def chunk_forward(q, k, v, g, beta, cu_seqlens, S0=None, chunk=64, scale=1.0):
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    T, H_qk, d_k = q.shape
    _, H_v, d_v = v.shape
    r = H_v // H_qk
    N = len(cu_seqlens) - 1
    o = np.zeros((T, H_v, d_v))
    Sf = np.zeros((N, H_v, d_v, d_k))
    for n in range(N):
        s0, s1 = int(cu_seqlens[n]), int(cu_seqlens[n + 1])
        for h in range(H_v):
            j = h // r
            S = np.zeros((d_v, d_k)) if S0 is None else np.array(S0[n, h], dtype=np.float64)
            for cs in range(s0, s1, chunk):
                ce = min(cs + chunk, s1)
                Q = l2n(q[cs:ce, j]) * scale
                K = l2n(k[cs:ce, j])
                V = v[cs:ce, h]
                G = np.cumsum(g[cs:ce, h])
                bt = beta[cs:ce, h]
                L = ce - cs
                diff = G[:, None] - G[None, :]
                incl = np.tril(np.ones((L, L), dtype=bool))
                Gam = np.where(incl, np.exp(np.where(incl, diff, 0.0)), 0.0)
                A = np.tril(bt[:, None] * Gam * (K @ K.T), -1)
                Tm = np.linalg.inv(np.eye(L) + A)
                U = Tm @ (bt[:, None] * V)
                W = Tm @ ((bt * np.exp(G))[:, None] * K)
                Vn = U - W @ S.T
                O = (np.exp(G)[:, None] * Q) @ S.T + ((Q @ K.T) * Gam) @ Vn
                S = np.exp(G[-1]) * S + Vn.T @ (np.exp(G[-1] - G)[:, None] * K)
                o[cs:ce, h] = O
            Sf[n, h] = S
    return o, Sf
