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


# ------------------------------------------------------------ prefill into the pool --

PREFILL_IMPLS = ["GDN_IMPL_AUTO", "GDN_IMPL_TENSOR_CORE_WHOLE_ROWS", "GDN_IMPL_TENSOR_CORE_SPLIT",
                 "GDN_IMPL_CUDA_CORE"]


@pytest.mark.parametrize("impl", PREFILL_IMPLS)
def test_prefill_slots_against_oracle(impl):
    """Sequences start from their slot (or zeros where has_initial_state is 0, or for slot
    -1), write their final state back in place; unnamed slots come back bit for bit."""
    from linear_attention_sequence_delta_b200 import gdn, gdn_prefill_slots
    from linear_attention_sequence_delta_b200.inputs import make_prefill_inputs
    lens = [70, 0, 130, 64, 1]
    P = make_prefill_inputs(lens, H_qk=2, H_v=4, d_k=128, d_v=128, seed=21)
    D = make_decode_inputs(steps=1, num_seqs=9, H_qk=2, H_v=4, d_k=128, d_v=128, seed=22)
    pool = D.state.contiguous()
    slots = torch.tensor([6, 2, -1, 0, 8], dtype=torch.int32)
    has_init = torch.tensor([1, 0, 1, 1, 0], dtype=torch.int32)
    Pd = P.to("cuda")
    pool_d = pool.cuda()
    o = gdn_prefill_slots(Pd.q, Pd.k, Pd.v, Pd.a, Pd.b, Pd.A_log, Pd.dt_bias, Pd.cu_seqlens,
                          pool_d, slots.cuda(), has_init.cuda(), impl=getattr(gdn, impl))
    assert gdn_sync_status() == 0
    cu = P.cu_seqlens.tolist()
    for n in range(len(lens)):
        s, use = int(slots[n]), bool(has_init[n]) and int(slots[n]) >= 0
        S0 = pool[s:s + 1].unsqueeze(0)[0] if use else torch.zeros(1, 4, 128, 128)
        o_ref, S_ref = oracle.forward(P.q[cu[n]:cu[n + 1]], P.k[cu[n]:cu[n + 1]],
                                      P.v[cu[n]:cu[n + 1]], P.a[cu[n]:cu[n + 1]],
                                      P.b[cu[n]:cu[n + 1]], P.A_log, P.dt_bias, [0, lens[n]], S0)
        if lens[n]:
            assert rel_err(o[cu[n]:cu[n + 1]], o_ref) <= TOL_BF16, n
        if s >= 0:
            assert rel_err(pool_d[s], S_ref[0]) <= TOL_BF16, n
    named = {int(x) for x in slots if x >= 0}
    rest = [i for i in range(9) if i not in named]
    assert torch.equal(pool_d[rest].cpu(), pool[rest])


def test_prefill_slots_then_decode_slots_equals_one_prefill():
    """A prefill into the pool followed by decode steps from it equals one longer prefill."""
    from linear_attention_sequence_delta_b200 import gdn_prefill, gdn_prefill_slots
    from linear_attention_sequence_delta_b200.inputs import make_prefill_inputs
    L0, steps = 100, 3
    P = make_prefill_inputs([L0 + steps] * 2, H_qk=2, H_v=4, d_k=128, d_v=128, seed=23)
    Pd = P.to("cuda")
    o_all, S_all = gdn_prefill(Pd.q, Pd.k, Pd.v, Pd.a, Pd.b, Pd.A_log, Pd.dt_bias, Pd.cu_seqlens,
                               None)
    idx = torch.cat([torch.arange(n * (L0 + steps), n * (L0 + steps) + L0) for n in range(2)])
    sub = lambda x: x[idx.cuda()].contiguous()
    cu = torch.tensor([0, L0, 2 * L0], dtype=torch.int32, device="cuda")
    pool = torch.zeros(4, 4, 128, 128, device="cuda")
    slots = torch.tensor([3, 1], dtype=torch.int32, device="cuda")
    gdn_prefill_slots(sub(Pd.q), sub(Pd.k), sub(Pd.v), sub(Pd.a), sub(Pd.b), Pd.A_log, Pd.dt_bias,
                      cu, pool, slots, torch.zeros(2, dtype=torch.int32, device="cuda"))
    tok = torch.tensor([[n * (L0 + steps) + L0 + s for s in range(steps)] for n in range(2)],
                       device="cuda")
    g = lambda x: x[tok].contiguous()
    o_d, _ = gdn_decode_slots(g(Pd.q), g(Pd.k), g(Pd.v), g(Pd.a), g(Pd.b), Pd.A_log, Pd.dt_bias,
                              pool, slots)
    assert gdn_sync_status() == 0
    assert rel_err(o_d, o_all[tok].cpu().float().numpy()) <= TOL_BF16
    assert rel_err(pool[slots.long()], S_all.cpu().numpy()) <= TOL_BF16


def test_prefill_bad_slot_reported():
    from linear_attention_sequence_delta_b200 import gdn_prefill_slots
    from linear_attention_sequence_delta_b200.inputs import make_prefill_inputs
    P = make_prefill_inputs([40, 20], H_qk=1, H_v=2, d_k=128, d_v=128, seed=24).to("cuda")
    pool = torch.zeros(2, 2, 128, 128, device="cuda")
    gdn_prefill_slots(P.q, P.k, P.v, P.a, P.b, P.A_log, P.dt_bias, P.cu_seqlens, pool,
                      torch.tensor([0, 5], dtype=torch.int32, device="cuda"))
    assert gdn_sync_status() == 7
    assert torch.all(pool[1] == 0)
    assert gdn_sync_status() == 0
