"""Helpers for GPU-vs-oracle parity tests (test infrastructure)."""
import numpy as np
import torch

import oracle

TOL_BF16 = 1e-2   # max|gpu - oracle| / max|oracle|, bf16 q/k/v/o
TOL_FP32 = 1e-4   # same, fp32 q/k/v/o


def rel_err(gpu, ref) -> float:
    g = gpu.detach().float().cpu().numpy().astype(np.float64) if hasattr(gpu, "detach") else gpu
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref).max()
    return float(np.abs(g - ref).max() / (den if den > 0 else 1.0))


def oracle_prefill_heads(P, heads, seqs=None, scale=1.0):
    """Oracle outputs for selected V heads (and optionally selected sequences).

    Returns {(n, h): (o [len, d_v], final [d_v, d_k])}. Each (sequence, head) unit
    is independent, so a sample is computed exactly as in the full run.
    """
    cu = P.cu_seqlens.cpu().numpy().astype(np.int64)
    N = len(cu) - 1
    seqs = range(N) if seqs is None else seqs
    H_qk, H_v = P.q.shape[1], P.v.shape[1]
    r = H_v // H_qk
    out = {}
    for n in seqs:
        s0, s1 = int(cu[n]), int(cu[n + 1])
        for h in heads:
            j = h // r
            S0 = None if P.initial_state is None else P.initial_state[n:n + 1, h:h + 1].cpu()
            o, Sf = oracle.forward(P.q[s0:s1, j:j + 1].cpu(), P.k[s0:s1, j:j + 1].cpu(),
                                   P.v[s0:s1, h:h + 1].cpu(), P.a[s0:s1, h:h + 1].cpu(),
                                   P.b[s0:s1, h:h + 1].cpu(), P.A_log[h:h + 1].cpu(),
                                   P.dt_bias[h:h + 1].cpu(), [0, s1 - s0], S0, scale=scale)
            out[(n, h)] = (o[:, 0], Sf[0, 0])
    return out


def oracle_mixer(P, eps=1e-6, scale=1.0):
    """The mixer core composed from the oracle's steps: the causal conv1d + SiLU over the
    q | k | v channels (the conv cache in and out), its output rounded to the I/O type as
    the API states, split into q, k and v heads, the gated delta rule, then the gated
    RMSNorm with z. Returns (y, final_state, conv_state_out)."""
    cu = P.cu_seqlens.cpu().numpy().astype(np.int64)
    T, C = P.x.shape
    H_v, d = P.z.shape[1], P.z.shape[2]
    H_qk = P.H_qk
    yc, so = oracle.conv1d_silu(P.x, P.conv_weight, P.conv_bias, cu, P.conv_state)
    yc = torch.from_numpy(yc).to(P.x.dtype)  # the post-conv q, k, v in the I/O type
    q = yc[:, :H_qk * d].reshape(T, H_qk, d)
    k = yc[:, H_qk * d:2 * H_qk * d].reshape(T, H_qk, d)
    v = yc[:, 2 * H_qk * d:].reshape(T, H_v, d)
    o, Sf = oracle.forward(q, k, v, P.a, P.b, P.A_log, P.dt_bias, cu, P.initial_state,
                           scale=scale)
    y = oracle.rmsnorm_gated(o, P.z, P.norm_weight, eps)
    return y, Sf, so
