"""gdn_decode_slots against the fp64 oracle: states in a pool of cache slots ("Qwen3.5
observation notes", section "Cache"), several tokens per sequence in one call with the
state after every token written out (draft verification, "Qwen3.5-MoE-35B-A3B
architecture teardown", section 6.2).

The oracle runs each sequence's L tokens as one packed prefill from the state found in
its slot (packing and decode = prefill are pinned for the oracle); the slot bookkeeping
itself is plain indexing. Tolerance as for the other paths: max|Δ|/max|ref| <= 1e-2
(bf16 I/O) and 1e-4 (fp32 I/O) on o, on the new pool states and on every intermediate
state; pool slots that no sequence names must come back bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_sequence_delta_b200 import (gdn_decode_slots, gdn_decode_step,
                                                  gdn_sync_status)
from linear_attention_sequence_delta_b200.inputs import make_decode_inputs
from tests.parity_util import TOL_BF16, TOL_FP32, rel_err

pytestmark = pytest.mark.gpu


def _inputs(N, L, num_slots, H_qk, H_v, d, dtype, seed):
    """Token inputs [N, L, ...] for N sequences and a pool of num_slots states."""
    D = make_decode_inputs(steps=L, num_seqs=num_slots, H_qk=H_qk, H_v=H_v, d_k=d, d_v=d,
                           io_dtype=dtype, seed=seed)
    tok = lambda x: x[:, :N].transpose(0, 1).contiguous()  # [L, N, ...] -> [N, L, ...]
    return (tok(D.q), tok(D.k), tok(D.v), tok(D.a), tok(D.b), D.A_log, D.dt_bias,
            D.state.contiguous())


def _oracle(q, k, v, a, b, A_log, dt_bias, pool, slots, scale=1.0):
    """Per live sequence: o [L, H_v, d], final state, and the states after each token."""
    N, L = q.shape[:2]
    out = {}
    for n in range(N):
        s = int(slots[n])
        if s < 0:
            continue
        S0 = pool[s:s + 1]
        o, Sf = oracle.forward(q[n], k[n], v[n], a[n], b[n], A_log, dt_bias, [0, L], S0,
                               scale=scale)
        inter = [oracle.forward(q[n, :t + 1], k[n, :t + 1], v[n, :t + 1], a[n, :t + 1],
                                b[n, :t + 1], A_log, dt_bias, [0, t + 1], S0, scale=scale)[1][0]
                 for t in range(L)]
        out[n] = (o, Sf[0], np.stack(inter))
    return out


def _slots(N, num_slots, pad, seed):
    g = torch.Generator().manual_seed(seed)
    s = torch.randperm(num_slots, generator=g)[:N].to(torch.int32)
    for i in pad:
        s[i] = -1
    return s


@pytest.mark.parametrize("dtype,d,L", [(torch.bfloat16, 128, 1), (torch.bfloat16, 128, 4),
                                       (torch.float32, 64, 3), (torch.bfloat16, 64, 16)])
def test_slots_multi_token_with_intermediates(dtype, d, L):
    N, num_slots, H_qk, H_v = 6, 11, 2, 4
    q, k, v, a, b, A_log, dt_bias, pool = _inputs(N, L, num_slots, H_qk, H_v, d, dtype,
                                                  seed=L + d)
    slots = _slots(N, num_slots, pad=[2], seed=d)
    pool_d = pool.cuda()
    o, inter = gdn_decode_slots(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), A_log.cuda(),
                                dt_bias.cuda(), pool_d, slots.cuda(), want_intermediate=True)
    assert gdn_sync_status() == 0
    tol = TOL_BF16 if dtype == torch.bfloat16 else TOL_FP32
    ref = _oracle(q, k, v, a, b, A_log, dt_bias, pool, slots)
    for n, (o_ref, S_ref, I_ref) in ref.items():
        s = int(slots[n])
        assert rel_err(o[n], o_ref) <= tol, n
        assert rel_err(pool_d[s], S_ref) <= tol, n
        assert rel_err(inter[n], I_ref) <= tol, n
        assert torch.equal(inter[n, L - 1], pool_d[s])
    assert torch.all(o[2] == 0)                        # the padding entry
    untouched = sorted(set(range(num_slots)) - {int(x) for x in slots if x >= 0})
    assert torch.equal(pool_d[untouched].cpu(), pool[untouched])


def test_single_token_identity_slots_equals_decode_step():
    """L = 1 without slots is gdn_decode_step (both within tolerance of the oracle)."""
    N, H_qk, H_v, d = 16, 4, 8, 128
    q, k, v, a, b, A_log, dt_bias, pool = _inputs(N, 1, N, H_qk, H_v, d, torch.bfloat16, seed=5)
    p1, p2 = pool.cuda(), pool.cuda()
    o1, _ = gdn_decode_slots(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), A_log.cuda(),
                             dt_bias.cuda(), p1)
    o2 = gdn_decode_step(q[:, 0].cuda(), k[:, 0].cuda(), v[:, 0].cuda(), a[:, 0].cuda(),
                         b[:, 0].cuda(), A_log.cuda(), dt_bias.cuda(), p2)
    assert gdn_sync_status() == 0
    o_ref, S_ref = oracle.decode_step(q[:, 0], k[:, 0], v[:, 0], a[:, 0], b[:, 0], A_log,
                                      dt_bias, pool)
    assert rel_err(o1[:, 0], o_ref) <= TOL_BF16 and rel_err(o2, o_ref) <= TOL_BF16
    assert rel_err(p1, S_ref) <= TOL_BF16 and rel_err(p2, S_ref) <= TOL_BF16
    # same arithmetic up to the order of the two norms' sums: far inside the tolerance
    assert rel_err(p1, p2.cpu().numpy()) <= 1e-5


def test_chained_calls_equal_one_multi_token_call():
    """Two calls of L = 2 from the pool equal one call of L = 4 (within fp32 rounding)."""
    N, H_qk, H_v, d = 3, 2, 4, 128
    q, k, v, a, b, A_log, dt_bias, pool = _inputs(N, 4, 5, H_qk, H_v, d, torch.float32, seed=9)
    slots = torch.tensor([4, 0, 2], dtype=torch.int32).cuda()
    cu = lambda x: x.cuda()
    p1, p2 = pool.cuda(), pool.cuda()
    o_all, _ = gdn_decode_slots(cu(q), cu(k), cu(v), cu(a), cu(b), cu(A_log), cu(dt_bias), p1,
                                slots)
    h = lambda x, i: x[:, 2 * i:2 * i + 2].contiguous().cuda()
    oa, _ = gdn_decode_slots(h(q, 0), h(k, 0), h(v, 0), h(a, 0), h(b, 0), cu(A_log),
                             cu(dt_bias), p2, slots)
    ob, _ = gdn_decode_slots(h(q, 1), h(k, 1), h(v, 1), h(a, 1), h(b, 1), cu(A_log),
                             cu(dt_bias), p2, slots)
    assert gdn_sync_status() == 0
    assert rel_err(torch.cat([oa, ob], 1), o_all.cpu().numpy()) <= 1e-6
    assert rel_err(p2, p1.cpu().numpy()) <= 1e-6


def test_bad_slot_reported_and_skipped():
    N, H_qk, H_v, d = 2, 2, 4, 64
    q, k, v, a, b, A_log, dt_bias, pool = _inputs(N, 2, 3, H_qk, H_v, d, torch.bfloat16, seed=3)
    pool_d = pool.cuda()
    slots = torch.tensor([1, 7], dtype=torch.int32).cuda()  # 7 >= 3 slots
    gdn_decode_slots(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), A_log.cuda(),
                     dt_bias.cuda(), pool_d, slots)
    assert gdn_sync_status() == 7
    assert torch.equal(pool_d[[0, 2]].cpu(), pool[[0, 2]])
    assert gdn_sync_status() == 0
