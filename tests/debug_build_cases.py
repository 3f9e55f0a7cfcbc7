"""Cases for the debug build, run by tests/test_debug_build_gpu.py in a process of its own
that loads libgdn_debug.so (GDN_LIBRARY): the tensor-core prefill's schedules on ragged
and empty sequences, more preparation units than workers, pool slots with padding entries, the mixer core with the
convolution and the norm fused in, and a call with one injected index check. Each call is
compared with the oracle, and the status word and the first failed check's site are read
after it. Prints one JSON list of {case, err, status, site} (test infrastructure).

    GDN_LIBRARY=.../libgdn_debug.so python -m tests.debug_build_cases
"""
import json

import numpy as np
import torch

import oracle
from linear_attention_sequence_delta_b200 import (gdn, gdn_mixer_prefill, gdn_prefill,
                                                  gdn_prefill_slots, gdn_sync_status)
from linear_attention_sequence_delta_b200.inputs import (make_mixer_prefill_inputs,
                                                         make_prefill_inputs)
from tests.parity_util import oracle_mixer, rel_err


def _prefill(P, impl, fault=gdn.GDN_FAULT_NONE):
    Pd = P.to("cuda")
    o, Sf = gdn_prefill(Pd.q, Pd.k, Pd.v, Pd.a, Pd.b, Pd.A_log, Pd.dt_bias, Pd.cu_seqlens,
                        Pd.initial_state, impl=impl, fault=fault)
    o_ref, S_ref = oracle.forward(P.q, P.k, P.v, P.a, P.b, P.A_log, P.dt_bias,
                                  P.cu_seqlens.numpy(), P.initial_state)
    return max(rel_err(o, o_ref), rel_err(Sf, S_ref))


def _slots():
    lens = [70, 0, 129, 5, 64]
    P = make_prefill_inputs(lens, H_qk=2, H_v=4, d_k=128, d_v=128, seed=41)
    g = torch.Generator().manual_seed(42)
    pool = torch.randn(6, 4, 128, 128, generator=g) * 0.05
    slots = torch.tensor([4, 0, -1, 2, 5], dtype=torch.int32)
    has_init = torch.tensor([1, 0, 1, 1, 0], dtype=torch.int32)
    Pd = P.to("cuda")
    pool_d = pool.cuda()
    o = gdn_prefill_slots(Pd.q, Pd.k, Pd.v, Pd.a, Pd.b, Pd.A_log, Pd.dt_bias, Pd.cu_seqlens,
                          pool_d, slots.cuda(), has_init.cuda(), impl=gdn.GDN_IMPL_TENSOR_CORE)
    cu = P.cu_seqlens.tolist()
    err = 0.0
    for n in range(len(lens)):
        s, use = int(slots[n]), bool(has_init[n]) and int(slots[n]) >= 0
        S0 = pool[s:s + 1].unsqueeze(0)[0] if use else torch.zeros(1, 4, 128, 128)
        sl = slice(cu[n], cu[n + 1])
        o_ref, S_ref = oracle.forward(P.q[sl], P.k[sl], P.v[sl], P.a[sl], P.b[sl], P.A_log,
                                      P.dt_bias, [0, cu[n + 1] - cu[n]], S0)
        if cu[n + 1] > cu[n]:
            err = max(err, rel_err(o[sl], o_ref))
        if s >= 0:
            err = max(err, rel_err(pool_d[s:s + 1], S_ref))
    return err


def _mixer(lens, impl):
    P = make_mixer_prefill_inputs(lens, H_qk=2, H_v=4, d=128, state_std=0.05, seed=43)
    Pd = P.to("cuda")
    cout = torch.empty_like(Pd.conv_state)
    y, Sf = gdn_mixer_prefill(Pd.x, Pd.conv_weight, Pd.conv_bias, Pd.cu_seqlens, Pd.a, Pd.b,
                              Pd.A_log, Pd.dt_bias, Pd.z, Pd.norm_weight, H_qk=P.H_qk,
                              conv_state_in=Pd.conv_state.clone(), conv_state_out=cout,
                              initial_state=Pd.initial_state, impl=impl)
    y_ref, S_ref, c_ref = oracle_mixer(P)
    exact = bool(np.array_equal(cout.float().cpu().numpy(), c_ref))
    return max(rel_err(y, y_ref), rel_err(Sf, S_ref), 0.0 if exact else 1.0)


def main():
    assert gdn.debug_build(), "the debug library is not the one loaded"
    ragged = make_prefill_inputs([70, 0, 1, 64, 129, 0, 5], H_qk=2, H_v=4, d_k=128, d_v=128,
                                 state_std=0.05, seed=44)
    many = make_prefill_inputs([100] * 8, H_qk=16, H_v=32, d_k=128, d_v=128, state_std=0.05,
                               seed=45)
    # more (chunk, QK head) units than preparation workers, over many short sequences: each
    # worker looks the next unit up (often across several sequence boundaries) and fetches
    # its rows and gate inputs one unit ahead
    rng = np.random.default_rng(47)
    units = make_prefill_inputs([int(x) for x in rng.integers(1, 300, size=96)], H_qk=8, H_v=32,
                                d_k=128, d_v=128, state_std=0.05, seed=48)
    cases = [
        ("ragged_half_rows", lambda: _prefill(ragged, gdn.GDN_IMPL_TENSOR_CORE)),
        ("ragged_whole_rows", lambda: _prefill(ragged, gdn.GDN_IMPL_TENSOR_CORE_WHOLE_ROWS)),
        ("ragged_split", lambda: _prefill(ragged, gdn.GDN_IMPL_TENSOR_CORE_SPLIT)),
        ("many_chains_auto", lambda: _prefill(many, gdn.GDN_IMPL_AUTO)),
        ("many_units_split", lambda: _prefill(units, gdn.GDN_IMPL_TENSOR_CORE_SPLIT)),
        ("slots_padding", _slots),
        ("mixer_auto", lambda: _mixer([70, 1, 129, 0, 33], gdn.GDN_IMPL_AUTO)),
        ("mixer_fused", lambda: _mixer([70, 1, 129, 0, 33], gdn.GDN_IMPL_TENSOR_CORE)),
        ("mixer_split", lambda: _mixer([70, 1, 129, 0, 33], gdn.GDN_IMPL_TENSOR_CORE_SPLIT)),
        ("inject_split", lambda: _prefill(ragged, gdn.GDN_IMPL_TENSOR_CORE_SPLIT,
                                          gdn.GDN_FAULT_BAD_INDEX)),
        ("inject_overlapped", lambda: _prefill(ragged, gdn.GDN_IMPL_TENSOR_CORE,
                                               gdn.GDN_FAULT_BAD_INDEX)),
        ("after_injection", lambda: _prefill(ragged, gdn.GDN_IMPL_TENSOR_CORE_SPLIT)),
    ]
    out = []
    for name, fn in cases:
        err = fn()
        site = gdn.debug_bad_index_site()
        status = gdn_sync_status()
        out.append(dict(case=name, err=float(err), status=int(status), site=int(site)))
    print(json.dumps(out))


if __name__ == "__main__":
    main()
