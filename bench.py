"""Benchmark of the Gated DeltaNet token mixer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on rank 0. A "step" is one gdn_prefill call on the largest single-GPU
workload, the packed varlen batch: 64 sequences with lengths ~ U[128, 8192] (274,156
tokens with seed 0), 16 QK / 32 V heads, d=128, bf16 q/k/v/o, fp32 gates, initial
states ~ N(0, 0.02^2) in, final states out. `value` is prefill tokens/s over the
whole job (all ranks; each rank runs its own copy of the workload, so scaling is
weak). The same line carries the other prefill workloads (the 35B-A3B layer, B=1,
T=4096, 32 V heads; the 397B-A17B long prefill, 4 x 16384 tokens, 64 V heads) under
"prefill_other_configs", the decode measurement (256 sequences x 64 V heads, 1000
consecutive in-place steps of gdn_decode_step) under "decode", the decode variants
and the steps around the delta rule.

Timing: W untimed warm-up steps; then K steps, each preceded by an L2 flush (a 512
MiB write, outside the timed window; the inputs, 4.7 GB, exceed L2 as well) and
bracketed by CUDA events on the launching stream; a barrier and a device synchronise
on both sides of the timed region; the max over ranks. `e2e` repeats the headline
prefill through the public Python API from pinned host buffers, host<->device copies
inside the timing. The CPU baseline is the fp64 oracle (test infrastructure) timed on
this host on a bounded sample of the same workload.

`roofline` is that of the dominant kernel of the step (the longest of the call's
launches): its duration comes from a kernel timer (CUDA events recorded around each
launch on the launching stream, every timed step), its algorithmic bytes are the
ones that kernel must move (see kernel_bytes), `traffic` is the DRAM bytes per launch
from the committed ncu record (profiles/roofline_traffic.json), null when that record
was taken on another build of the kernel. `roofline.step` gives the whole call
against the slower of the HBM and tensor roofs.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "varlen_64"
WORKLOAD_DESC = ("varlen_64: 64 sequences, lengths ~ U[128, 8192] packed via cu_seqlens, "
                 "H_qk=16, H_v=32, d=128, bf16 q/k/v/o, fp32 gates, initial states "
                 "~N(0, 0.02^2) in, final states out")
OTHER_PREFILL = ("prefill_35b", "prefill_397b_long")
METRIC = "GDN prefill tokens/s and decode steps/s on 1 B200, % of roofline"
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "roofline_traffic.json")
TC_SOURCE = os.path.join(ROOT, "linear_attention_sequence_delta_b200", "csrc",
                         "gdn_prefill_tc.cu")


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(
            p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def prefill_bytes(T, N, H_qk, H_v, d, io_bytes, with_initial):
    """Algorithmic HBM bytes of one gdn_prefill call: q, k, v read, o written,
    a and b read, the final state written (and the initial state read if given)."""
    b = 2 * T * H_qk * d * io_bytes + 2 * T * H_v * d * io_bytes + 2 * T * H_v * 4
    b += N * H_v * d * d * 4 * (2 if with_initial else 1)
    return b


def kernel_bytes(kernel, T, N, H_qk, H_v, d, io_bytes, with_initial):
    """Algorithmic HBM bytes of one launch of a kernel of the tensor-core prefill:
    the one-launch kernels move the whole call's; the chain reads q, k, v, writes o
    and the final states (and reads the initial ones); the prep reads q, k, a and b
    (its records are intermediates, not algorithmic bytes)."""
    if kernel.startswith("fused"):
        return prefill_bytes(T, N, H_qk, H_v, d, io_bytes, with_initial)
    if kernel == "chain":
        return prefill_bytes(T, N, H_qk, H_v, d, io_bytes, with_initial) - 2 * T * H_v * 4
    if kernel == "prep":
        return 2 * T * H_qk * d * io_bytes + 2 * T * H_v * 4
    return 4 * (N + 1)


def prefill_flops(T, N, H_qk, H_v, d, C=64):
    """Algorithmic tensor flops of the chunk form per token: the in-chunk products
    K K^T and Q K^T once per QK head (4 C d), and per V head the solve-applied value
    update (2 C d), the intra-chunk P V_new and S0 [K; Q]^T products (4 C d) and the
    state's three chunk products (6 d^2)."""
    return T * (H_qk * 4 * C * d + H_v * (2 * C * d + 4 * C * d + 6 * d * d))


def _source_sha1(path=TC_SOURCE):
    """SHA-1 of the kernel source's code: comments removed and every run of blank space
    turned into one space, so that a traffic record stays valid across edits of comments
    and layout only."""
    import re
    with open(path, encoding="utf-8") as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    src = re.sub(r"\s+", " ", src).strip()
    return hashlib.sha1(src.encode()).hexdigest()


def run_metadata(dev):
    """Where the number was measured: the GPU (name, SM count, memory, driver and CUDA
    runtime of the process), the library that ran (a hash of the kernel sources and
    the public header, whether it is the debug build) and, where the checkout has its
    history, the git commit."""
    from linear_attention_sequence_delta_b200 import gdn
    props = torch.cuda.get_device_properties(dev)
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "linear_attention_sequence_delta_b200", "csrc")
    files = [os.path.join(csrc, f) for f in sorted(os.listdir(csrc)) if f.endswith((".cu", ".cuh"))]
    for path in files + [os.path.join(ROOT, "include", "gdn.h")]:
        with open(path, "rb") as f:
            h.update(f.read())
    try:
        sha = subprocess.run(["git", "-C", ROOT, "rev-parse", "HEAD"], capture_output=True,
                             text=True, timeout=10).stdout.strip() or None
    except Exception:
        sha = None
    try:
        import pynvml
        pynvml.nvmlInit()
        driver = pynvml.nvmlSystemGetDriverVersion()
        driver = driver.decode() if isinstance(driver, bytes) else driver
    except Exception:
        driver = None
    return {"gpu": {"name": props.name, "sm_count": props.multi_processor_count,
                    "memory_gib": round(props.total_memory / 2**30, 1),
                    "driver": driver, "torch_cuda": torch.version.cuda},
            "library": {"sources_sha1": h.hexdigest(), "debug_build": gdn.debug_build(),
                        "git_sha": sha}}


def kernel_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu record,
    or None (no record, or one taken on another build of the kernel source)."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)[f"{kernel}@{workload}"]
        if rec["kernel_source_sha1"] != _source_sha1():
            return None
        return int(rec["traffic_bytes_per_launch"])
    except Exception:
        return None


def decode_bytes(N, H_qk, H_v, d, io_bytes):
    return 2 * N * H_v * d * d * 4 + N * (2 * H_qk * d + 2 * H_v * d) * io_bytes + 2 * N * H_v * 4


def mixer_bytes(T, N, C, K, rows, d, io_bytes, N_dec, C_dec):
    """Algorithmic HBM bytes of the steps around the delta rule: the conv reads x and
    writes y (plus the taps and, per sequence, the K-1 cached positions written out);
    the conv decode reads x, the taps and the cache and writes y and the slid cache; the
    gated norm reads o and z and writes y (plus the d-long weight)."""
    conv = 2 * T * C * io_bytes + C * K * 4 + N * (K - 1) * C * io_bytes
    conv_dec = 2 * N_dec * C_dec * io_bytes + C_dec * K * 4 + 2 * N_dec * (K - 1) * C_dec * io_bytes
    norm = 3 * rows * d * io_bytes + d * 4
    return conv, conv_dec, norm


def _time_op(fn, iters, flush, stream):
    """Mean device time of fn() over iters launches, the L2 flushed before each."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(iters)]
    for i in range(iters):
        flush.fill_(i & 0xFF)
        evs[i][0].record(stream)
        fn()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / iters


def run_mixer(rank, dev, flush, stream, hbm, peak_src, iters):
    """The convolution in front of the delta rule and the gated norm after it, on the
    35B-A3B layer (T=4096, conv_dim=8192, 32 V heads x 128) and the conv decode step on
    the 397B-A17B decode batch (256 sequences, conv_dim=12288)."""
    from linear_attention_sequence_delta_b200 import gdn
    from linear_attention_sequence_delta_b200.inputs import make_mixer_inputs
    M = make_mixer_inputs(num_seqs=1, seq_len=4096, H_qk=16, H_v=32, d_k=128, d_v=128,
                          seed=rank, device=dev)
    Md = make_mixer_inputs([1] * 256, H_qk=16, H_v=64, d_k=128, d_v=128, seed=rank,
                           device=dev)
    T, C = M.x.shape
    K = M.conv_weight.shape[1]
    y = torch.empty_like(M.x)
    cst = torch.empty_like(M.conv_state)
    yn = torch.empty_like(M.o)
    yd = torch.empty_like(Md.x)
    st_d = Md.conv_state.clone()
    conv_ms = _time_op(lambda: gdn.gdn_conv1d_silu(M.x, M.conv_weight, None, M.cu_seqlens, None,
                                                   out=y, conv_state_out=cst),
                       iters, flush, stream)
    dec_ms = _time_op(lambda: gdn.gdn_conv1d_silu_decode(Md.x, Md.conv_weight, None, st_d,
                                                         out=yd),
                      iters, flush, stream)
    norm_ms = _time_op(lambda: gdn.gdn_rmsnorm_gated(M.o, M.z, M.norm_weight, 1e-6, out=yn),
                       iters, flush, stream)
    rows, d = M.o.shape[0] * M.o.shape[1], M.o.shape[2]
    b_conv, b_dec, b_norm = mixer_bytes(T, 1, C, K, rows, d, 2, Md.x.shape[0], Md.x.shape[1])

    def roof(b, ms_):
        gbs = b / (ms_ / 1e3) / 1e9
        return {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                "algorithmic_bytes": b, "kernel_ms": ms_, "peak_source": peak_src}

    out = {
        "conv1d_silu": {"workload": f"T={T}, conv_dim={C}, K={K}, bf16, zero cache in, "
                                    "cache out", "tokens_per_s": T / (conv_ms / 1e3),
                        "roofline": roof(b_conv, conv_ms), "launches_per_call": 2},
        "conv1d_silu_decode": {"workload": f"{Md.x.shape[0]} seqs x 1 token, "
                                           f"conv_dim={Md.x.shape[1]}, K={K}, bf16, "
                                           "cache in place",
                               "us_per_step": dec_ms * 1e3, "roofline": roof(b_dec, dec_ms),
                               "launches_per_call": 1},
        "rmsnorm_gated": {"workload": f"{T} tokens x {M.o.shape[1]} V heads x {d}, bf16",
                          "tokens_per_s": T / (norm_ms / 1e3), "roofline": roof(b_norm, norm_ms),
                          "launches_per_call": 1},
        "l2": "flushed (512 MiB write) before every timed launch",
        "iters": iters,
    }
    return out, iters * 4


def mixer_call_bytes(T, N, H_qk, H_v, d, K, io_bytes, with_initial):
    """Algorithmic HBM bytes of one gdn_mixer_prefill call: x read, z read, y written
    (io_bytes each element), a and b read, the conv taps read, the conv cache read and
    written, the final states written (and the initial states read)."""
    C = (2 * H_qk + H_v) * d
    b = T * C * io_bytes + 2 * T * H_v * d * io_bytes + 2 * T * H_v * 4 + C * K * 4
    b += 2 * N * (K - 1) * C * io_bytes
    b += N * H_v * d * d * 4 * (2 if with_initial else 1)
    return b


def run_mixer_prefill(rank, dev, flush, stream, hbm, peak_src, iters):
    """gdn_mixer_prefill in its default schedule (the convolution, the tensor-core prefill
    reading the post-conv buffer, the norm in place) and in the fused one (conv1d + SiLU
    in the prefill's preparation, gated RMSNorm in the chain's output), against the same
    steps as separate calls: the conv of the q, k and v parts (dense tensors), gdn_prefill,
    gdn_rmsnorm_gated. On the 35B-A3B layer shape (T=4096) and the packed varlen batch
    (64 sequences)."""
    from linear_attention_sequence_delta_b200 import gdn
    from linear_attention_sequence_delta_b200.inputs import WORKLOADS, make_mixer_prefill_inputs
    out, launches = {}, 0
    timer = gdn.Timer()
    for name in ("prefill_35b", "varlen_64"):
        W = WORKLOADS[name]
        lens = "random" if W.get("lengths") == "random" else None
        P = make_mixer_prefill_inputs(lens, num_seqs=W["num_seqs"], seq_len=W.get("seq_len", 256),
                                      len_lo=W.get("len_lo", 128), len_hi=W.get("len_hi", 8192),
                                      H_qk=W["H_qk"], H_v=W["H_v"], d=W["d_k"],
                                      state_std=W.get("state_std"), seed=rank, device=dev)
        T, C = P.x.shape
        N, H_qk, H_v, d = P.num_seqs, P.H_qk, P.z.shape[1], P.z.shape[2]
        K = P.conv_weight.shape[1]
        y = torch.empty_like(P.z)
        Sf = torch.empty((N, H_v, d, d), device=dev, dtype=torch.float32)
        cout = torch.empty_like(P.conv_state)
        ws = torch.empty((gdn.mixer_workspace_size(N, T, H_qk, H_v, d),), device=dev,
                         dtype=torch.uint8)
        call = lambda tm=None, impl=gdn.GDN_IMPL_AUTO: gdn.gdn_mixer_prefill(
            P.x, P.conv_weight, P.conv_bias, P.cu_seqlens, P.a, P.b, P.A_log, P.dt_bias, P.z,
            P.norm_weight, H_qk=H_qk, conv_state_in=P.conv_state, conv_state_out=cout,
            initial_state=P.initial_state, out=y, final_state=Sf, workspace=ws, timer=tm,
            impl=impl)
        fused = lambda tm=None: call(tm, gdn.GDN_IMPL_TENSOR_CORE)
        # the separate steps on dense parts (q, k, v each its own [T, H d] tensor)
        bounds = [(0, H_qk * d), (H_qk * d, 2 * H_qk * d), (2 * H_qk * d, C)]
        xs = [P.x[:, a_:b_].contiguous() for a_, b_ in bounds]
        wsp = [P.conv_weight[a_:b_].contiguous() for a_, b_ in bounds]
        bsp = [P.conv_bias[a_:b_].contiguous() for a_, b_ in bounds]
        csp = [P.conv_state[:, :, a_:b_].contiguous() for a_, b_ in bounds]
        ys = [torch.empty_like(x_) for x_ in xs]
        cos = [torch.empty_like(c_) for c_ in csp]
        o = torch.empty_like(P.z)
        pws = torch.empty((gdn.workspace_size(N, T, H_qk, H_v, d, d),), device=dev,
                          dtype=torch.uint8)

        def steps():
            for x_, w_, b_, c_, y_, co_ in zip(xs, wsp, bsp, csp, ys, cos):
                gdn.gdn_conv1d_silu(x_, w_, b_, P.cu_seqlens, c_, out=y_, conv_state_out=co_)
            gdn.gdn_prefill(ys[0].view(T, H_qk, d), ys[1].view(T, H_qk, d), ys[2].view(T, H_v, d),
                            P.a, P.b, P.A_log, P.dt_bias, P.cu_seqlens, P.initial_state, out=o,
                            final_state=Sf, workspace=pws)
            gdn.gdn_rmsnorm_gated(o, P.z, P.norm_weight, 1e-6, out=y)

        ms_a = _time_op(call, iters, flush, stream)
        ms_f = _time_op(fused, iters, flush, stream)
        ms_s = _time_op(steps, iters, flush, stream)
        call(timer)
        ka = timer.times()
        fused(timer)
        kn = timer.times()
        launches += 3 * (iters + 3) * 6
        byts = mixer_call_bytes(T, N, H_qk, H_v, d, K, 2, P.initial_state is not None)
        out[name] = {
            "workload": f"N={N}, T_total={T}, H_qk={H_qk}, H_v={H_v}, d={d}, conv_dim={C}, K={K}, "
                        "bf16 x/z/y, conv cache in and out"
                        + (", initial states in" if P.initial_state is not None else "")
                        + ", final states out",
            "call_ms": ms_a, "call_kernels_ms": {k_: v_ for k_, v_ in ka},
            "fused_ms": ms_f, "fused_kernels_ms": {k_: v_ for k_, v_ in kn},
            "separate_steps_ms": ms_s,
            "separate_steps": "3 conv1d_silu (q, k, v parts) + gdn_prefill + gdn_rmsnorm_gated",
            "tokens_per_s": T / (ms_a / 1e3), "algorithmic_bytes": byts,
            "achieved_gbs": byts / (ms_a / 1e3) / 1e9,
            "frac_hbm": byts / (ms_a / 1e3) / 1e9 / hbm, "peak_source": peak_src}
        del P, y, Sf, cout, ws, xs, ys, o, pws
    timer.close()
    out["l2"] = "flushed (512 MiB write) before every timed call"
    out["iters"] = iters
    return out, launches


def run_decode_variants(rank, dev, flush, stream, hbm, peak_src, iters):
    """gdn_decode_slots on the 397B-A17B decode shape (256 sequences, 64 V heads, d=128):
    L = 1 with the states scattered over a pool of 512 slots (continuous batching), and
    L = 2 (a token plus one MTP draft) with the per-token states written out."""
    from linear_attention_sequence_delta_b200 import gdn
    from linear_attention_sequence_delta_b200.inputs import make_decode_inputs
    N, pool_n, H_qk, H_v, d = 256, 512, 16, 64, 128
    D = make_decode_inputs(steps=2, num_seqs=pool_n, H_qk=H_qk, H_v=H_v, d_k=d, d_v=d,
                           seed=rank, device=dev)
    g = torch.Generator(device="cpu").manual_seed(rank)
    slots = torch.randperm(pool_n, generator=g)[:N].to(torch.int32).to(dev)
    tok = lambda x, L: x[:L, :N].transpose(0, 1).contiguous()
    out = {}
    for L, inter in ((1, False), (2, True)):
        q, k, v, a, b = (tok(x, L) for x in (D.q, D.k, D.v, D.a, D.b))
        o = torch.empty((N, L, H_v, d), device=dev, dtype=q.dtype)
        I = torch.empty((N, L, H_v, d, d), device=dev, dtype=torch.float32) if inter else None
        ms = _time_op(lambda: gdn.gdn_decode_slots(q, k, v, a, b, D.A_log, D.dt_bias, D.state,
                                                   slots, out=o, intermediate_states=I),
                      iters, flush, stream)
        byts = (2 + (L if inter else 0)) * N * H_v * d * d * 4 \
            + N * L * (2 * H_qk * d + 2 * H_v * d) * 2 + 2 * N * L * H_v * 4 + N * 4
        gbs = byts / (ms / 1e3) / 1e9
        out[f"L{L}" + ("_intermediates" if inter else "")] = {
            "workload": f"{N} seqs x {L} token(s), states in a pool of {pool_n} slots, "
                        f"H_qk={H_qk}, H_v={H_v}, d={d}, bf16"
                        + (", state after every token written" if inter else ""),
            "us_per_call": ms * 1e3, "tokens_per_s": N * L / (ms / 1e3),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                         "frac": gbs / hbm, "algorithmic_bytes": byts, "kernel_ms": ms,
                         "peak_source": peak_src}}
    # the single-token step with the state stored in bf16 (half the state bytes)
    S16 = D.state[:N].to(torch.bfloat16)
    q, k, v, a, b = (x[0, :N].contiguous() for x in (D.q, D.k, D.v, D.a, D.b))
    o1 = torch.empty((N, H_v, d), device=dev, dtype=q.dtype)
    ms = _time_op(lambda: gdn.gdn_decode_step_bf16_state(q, k, v, a, b, D.A_log, D.dt_bias, S16,
                                                         out=o1), iters, flush, stream)
    byts = 2 * N * H_v * d * d * 2 + N * (2 * H_qk * d + 2 * H_v * d) * 2 + 2 * N * H_v * 4
    gbs = byts / (ms / 1e3) / 1e9
    out["L1_bf16_state"] = {
        "workload": f"{N} seqs x 1 token, H_qk={H_qk}, H_v={H_v}, d={d}, bf16 q/k/v/o, "
                    "bf16 state in place (dense, no slots)",
        "us_per_call": ms * 1e3, "tokens_per_s": N / (ms / 1e3),
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                     "frac": gbs / hbm, "algorithmic_bytes": byts, "kernel_ms": ms,
                     "peak_source": peak_src}}
    out["l2"] = "flushed (512 MiB write) before every timed launch"
    out["iters"] = iters
    return out, 3 * iters


def run_other_prefill(rank, dev, flush, stream, hbm, tc_burst, peak_src, iters,
                      names=OTHER_PREFILL, num_seqs=None):
    """gdn_prefill on the other prefill workloads: the 35B-A3B layer (B=1, T=4096,
    16 QK / 32 V heads; 32 chains, one overlapped launch) and the 397B-A17B long
    prefill (4 x 16384 tokens, 16 QK / 64 V heads; 256 chains, separate launches).
    Each call's kernels are timed by a kernel timer; the call itself with CUDA events
    around it, the L2 flushed before each call."""
    from linear_attention_sequence_delta_b200 import gdn
    from linear_attention_sequence_delta_b200.inputs import WORKLOADS, make_prefill_inputs
    out, launches = {}, 0
    timer = gdn.Timer()
    for name in names:
        if not name:
            continue
        wl = dict(WORKLOADS[name], **({"num_seqs": num_seqs} if num_seqs else {}))
        P = make_prefill_inputs(**wl, seed=rank, device=dev)
        T, H_qk, d = P.q.shape
        H_v, N = P.v.shape[1], P.num_seqs
        o = torch.empty((T, H_v, d), device=dev, dtype=P.q.dtype)
        Sf = torch.empty((N, H_v, d, d), device=dev, dtype=torch.float32)
        work = torch.empty((max(gdn.workspace_size(N, T, H_qk, H_v, d, d), 1),), device=dev,
                           dtype=torch.uint8)
        call = lambda tm=None: gdn.gdn_prefill(P.q, P.k, P.v, P.a, P.b, P.A_log, P.dt_bias,
                                               P.cu_seqlens, P.initial_state, out=o,
                                               final_state=Sf, workspace=work, timer=tm)
        ms = _time_op(call, iters, flush, stream)
        kms = {}
        for i in range(iters):
            flush.fill_(i & 0xFF)
            call(timer)
            for kn, t_ in timer.times():
                kms.setdefault(kn, []).append(t_)
        torch.cuda.synchronize()
        launches += (iters + 3) * len(kms) + iters * len(kms)
        with_init = P.initial_state is not None
        byts = prefill_bytes(T, N, H_qk, H_v, d, 2, with_initial=with_init)
        flops = prefill_flops(T, N, H_qk, H_v, d)
        t_roof = max(byts / (hbm * 1e9), flops / (tc_burst * 1e12))
        mean_k = {kn: sum(v_) / len(v_) for kn, v_ in kms.items()}
        dom = max(mean_k, key=mean_k.get)
        dom_b = kernel_bytes(dom, T, N, H_qk, H_v, d, 2, with_init)
        out[name] = {
            "workload": f"N={N}, T_total={T}, H_qk={H_qk}, H_v={H_v}, d={d}, bf16 q/k/v/o"
                        + (", initial states in" if with_init else "")
                        + ", final states out",
            "ms_per_call": ms, "tokens_per_s": T / (ms / 1e3),
            "kernels_ms": mean_k,
            "algorithmic_bytes": byts, "algorithmic_flops": flops,
            "achieved_gbs": byts / (ms / 1e3) / 1e9,
            "frac_hbm": byts / (ms / 1e3) / 1e9 / hbm,
            "frac_tensor": flops / (ms / 1e3) / 1e12 / tc_burst,
            "frac_of_slower_roof": t_roof / (ms / 1e3),
            "dominant_kernel": {"kernel": dom, "kernel_ms": mean_k[dom],
                                "algorithmic_bytes": dom_b,
                                "frac_hbm": dom_b / (mean_k[dom] / 1e3) / 1e9 / hbm,
                                "traffic": kernel_traffic(dom, name)},
            "peak_source": peak_src}
        del P, o, Sf, work
    timer.close()
    out["l2"] = "flushed (512 MiB write) before every timed call"
    out["iters"] = iters
    return out, launches


class Clocks:
    """nvidia-smi sampled every 200 ms while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = [r.split(", ") for r in (getattr(self, "out", "") or "").strip().splitlines()]
        rows = [r for r in rows if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _max_over_ranks(x: float, ws: int, device) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def run_ours(args):
    from linear_attention_sequence_delta_b200 import gdn
    from linear_attention_sequence_delta_b200.inputs import (DECODE_STEPS, DECODE_WORKLOAD,
                                                             WORKLOADS, make_decode_inputs,
                                                             make_prefill_inputs)
    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    gdn.load_library()
    hbm, tc_burst, tc_sust, peak_src = _peaks()
    W = dict(WORKLOADS[WORKLOAD], **({"num_seqs": args.seqs} if args.seqs else {}))
    P = make_prefill_inputs(**W, seed=rank, device=dev)
    T, H_qk, d = P.q.shape
    H_v = P.v.shape[1]
    N = P.num_seqs
    o = torch.empty((T, H_v, d), device=dev, dtype=P.q.dtype)
    Sf = torch.empty((N, H_v, d, d), device=dev, dtype=torch.float32)
    wsz = gdn.workspace_size(N, T, H_qk, H_v, d, d)
    work = torch.empty((max(wsz, 1),), device=dev, dtype=torch.uint8)
    flush = torch.empty((512 << 20,), device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)
    timer = gdn.Timer()

    def step(tm=None):
        gdn.gdn_prefill(P.q, P.k, P.v, P.a, P.b, P.A_log, P.dt_bias, P.cu_seqlens,
                        P.initial_state, out=o, final_state=Sf, workspace=work, timer=tm)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = Clocks(local)
    kernel_ms = {}  # kernel name -> [ms per timed step]
    _barrier(ws)
    torch.cuda.synchronize()
    with clocks:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)  # L2 flush, outside the events
            ev[i][0].record(stream)
            step(timer)
            ev[i][1].record(stream)
            for name, kms in timer.times():  # waits for this step only
                kernel_ms.setdefault(name, []).append(kms)
        torch.cuda.synchronize()
        _barrier(ws)
        # ---- decode: 1000 consecutive steps on the 397B-A17B GDN shape ----
        dec = None
        if not args.no_decode:
            dw = dict(DECODE_WORKLOAD, num_seqs=args.decode_seqs)
            D = make_decode_inputs(steps=args.decode_steps, seed=rank, device=dev, **dw)
            od = torch.empty_like(D.v[0])
            for t in range(min(3, args.decode_steps)):  # warm-up on a copy of the state
                gdn.gdn_decode_step(D.q[t], D.k[t], D.v[t], D.a[t], D.b[t], D.A_log, D.dt_bias,
                                    D.state.clone(), out=od)
            torch.cuda.synchronize()
            _barrier(ws)
            d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            d0.record(stream)
            for t in range(args.decode_steps):
                gdn.gdn_decode_step(D.q[t], D.k[t], D.v[t], D.a[t], D.b[t], D.A_log, D.dt_bias,
                                    D.state, out=od)
            d1.record(stream)
            torch.cuda.synchronize()
            dec_ms = _max_over_ranks(d0.elapsed_time(d1), ws, dev)
            Nd, H_qkd, H_vd = D.q.shape[1], D.q.shape[2], D.v.shape[2]
            per_step_s = dec_ms / 1e3 / args.decode_steps
            db = decode_bytes(Nd, H_qkd, H_vd, d, 2)
            dec = {"value": ws * args.decode_steps / (dec_ms / 1e3), "unit": "steps/s",
                   "tokens_per_s": ws * Nd * args.decode_steps / (dec_ms / 1e3),
                   "steps": args.decode_steps, "us_per_step": per_step_s * 1e6,
                   "workload": f"decode: {Nd} seqs x 1 token, H_qk={H_qkd}, H_v={H_vd}, d={d}, "
                               "bf16 q/k/v/o, fp32 state ~N(0,0.02^2) in place",
                   "roofline": {"bound": "hbm", "achieved": db / per_step_s / 1e9,
                                "peak": hbm, "unit": "GB/s",
                                "frac": db / per_step_s / 1e9 / hbm, "traffic": None,
                                "algorithmic_bytes": db, "peak_source": peak_src},
                   "gpu_launches": args.decode_steps}
            del D
        mixer, mixer_launches = None, 0
        if not args.no_mixer:
            mixer, mixer_launches = run_mixer(rank, dev, flush, stream, hbm, peak_src,
                                              args.mixer_iters)
        dvar, dvar_launches = None, 0
        if not args.no_decode:
            dvar, dvar_launches = run_decode_variants(rank, dev, flush, stream, hbm, peak_src,
                                                      args.mixer_iters)
        mixp, mixp_launches = None, 0
        if not args.no_mixer:
            mixp, mixp_launches = run_mixer_prefill(rank, dev, flush, stream, hbm, peak_src,
                                                    args.other_iters)
        other, other_launches = None, 0
        if not args.no_other_prefill:
            other, other_launches = run_other_prefill(rank, dev, flush, stream, hbm, tc_burst,
                                                      peak_src, args.other_iters,
                                                      args.other_prefill.split(","),
                                                      args.other_prefill_seqs)
    kern_ms = [a.elapsed_time(b) for a, b in ev]
    ms = _max_over_ranks(sum(kern_ms) / len(kern_ms), ws, dev)
    tok_s = ws * T / (ms / 1e3)
    with_init = P.initial_state is not None
    byts = prefill_bytes(T, N, H_qk, H_v, d, 2, with_initial=with_init)
    flops = prefill_flops(T, N, H_qk, H_v, d)
    achieved = byts / (ms / 1e3) / 1e9
    t_roof = max(byts / (hbm * 1e9), flops / (tc_burst * 1e12))
    mean_k = {n_: _max_over_ranks(sum(v_) / len(v_), ws, dev) for n_, v_ in kernel_ms.items()}
    dom = max(mean_k, key=mean_k.get)
    dom_ms = mean_k[dom]
    dom_bytes = kernel_bytes(dom, T, N, H_qk, H_v, d, 2, with_init)

    e2e = None
    if not args.no_e2e:
        e2e = _e2e(args, P, o, Sf, ws, dev, stream)

    line = {
        "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC + f" ({N} sequences, {T} tokens per rank)",
                   "global_batch": ws * N, "seq_len": T, "parallelism": f"replicas x{ws}",
                   "l2": "flushed (512 MiB write) before every timed step; inputs exceed L2"},
        "roofline": {"bound": "hbm", "achieved": dom_bytes / (dom_ms / 1e3) / 1e9, "peak": hbm,
                     "unit": "GB/s", "frac": dom_bytes / (dom_ms / 1e3) / 1e9 / hbm,
                     "traffic": kernel_traffic(dom, WORKLOAD), "kernel": dom,
                     "algorithmic_bytes": dom_bytes, "kernel_ms": dom_ms,
                     "peak_source": peak_src, "kernels_ms": mean_k,
                     "step": {"algorithmic_bytes": byts, "achieved_gbs": achieved,
                              "frac_hbm": achieved / hbm, "algorithmic_flops": flops,
                              "achieved_tflops": flops / (ms / 1e3) / 1e12,
                              "peak_tflops": tc_burst,
                              "frac_tensor": flops / (ms / 1e3) / 1e12 / tc_burst,
                              "frac_of_slower_roof": t_roof / (ms / 1e3)}},
        "e2e": e2e,
        "gpu_launches": sum(len(v_) for v_ in kernel_ms.values()),
        "gpu_launches_other_blocks": (args.decode_steps if dec else 0) + mixer_launches
                                     + dvar_launches + other_launches + mixp_launches,
        "clocks": clocks.summary(),
        "prefill_other_configs": other,
        "decode": dec,
        "decode_slots": dvar,
        "mixer": mixer,
        "mixer_prefill": mixp,
        "run": run_metadata(dev),
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def _e2e(args, P, o, Sf, ws, dev, stream):
    """Prefill through the public API from pinned host buffers: every step copies its
    inputs host -> device, runs gdn_prefill and reads o and the final states back. The
    calls run in order on one stream; the copies run on a host-to-device and a
    device-to-host stream with two sets of buffers, so one step's read-back and the next
    step's upload overlap the current call, as a serving loop would run them."""
    from linear_attention_sequence_delta_b200 import gdn
    T = P.q.shape[0]
    names = ("q", "k", "v", "a", "b", "A_log", "dt_bias", "cu_seqlens", "initial_state")
    host = {k_: getattr(P, k_).cpu().pin_memory() for k_ in names
            if getattr(P, k_) is not None}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o.numel() * o.element_size() + Sf.numel() * Sf.element_size()
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    work = torch.empty((max(gdn.workspace_size(P.num_seqs, T, P.q.shape[1], P.v.shape[1],
                                               P.q.shape[2], P.v.shape[2]), 1),),
                       device=dev, dtype=torch.uint8)
    ev = lambda: torch.cuda.Event()
    sets = [{"dev": {k_: torch.empty_like(t, device=dev) for k_, t in host.items()},
             "o": torch.empty_like(o), "S": torch.empty_like(Sf),
             "o_h": torch.empty(o.shape, dtype=o.dtype).pin_memory(),
             "S_h": torch.empty(Sf.shape, dtype=Sf.dtype).pin_memory(),
             "in_ready": ev(), "in_free": ev(), "out_ready": ev(), "out_free": ev()}
            for _ in range(2)]
    for b_ in sets:  # both sets start free
        b_["in_free"].record(stream)
        b_["out_free"].record(stream)

    def e2e_step(i):
        b_ = sets[i & 1]
        with torch.cuda.stream(up):  # inputs of step i, once step i-2 stopped reading them
            up.wait_event(b_["in_free"])
            for k_, t in host.items():
                b_["dev"][k_].copy_(t, non_blocking=True)
            b_["in_ready"].record(up)
        stream.wait_event(b_["in_ready"])
        stream.wait_event(b_["out_free"])  # step i-2's outputs have been read back
        dv = b_["dev"]
        gdn.gdn_prefill(dv["q"], dv["k"], dv["v"], dv["a"], dv["b"], dv["A_log"],
                        dv["dt_bias"], dv["cu_seqlens"], dv.get("initial_state"), out=b_["o"],
                        final_state=b_["S"],
                        workspace=work)
        b_["in_free"].record(stream)
        b_["out_ready"].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(b_["out_ready"])
            b_["o_h"].copy_(b_["o"], non_blocking=True)
            b_["S_h"].copy_(b_["S"], non_blocking=True)
            b_["out_free"].record(down)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    _barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_stream(stream)
    down.wait_stream(stream)
    for i in range(args.steps):
        e2e_step(i)
    stream.wait_stream(up)
    stream.wait_stream(down)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(e0.elapsed_time(e1) / args.steps, ws, dev)
    return {"value": ws * T / (e2e_ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
            "copy_streams": 2}


def _reference_sample(seed=0, min_tokens=8192):
    """A bounded sample of the headline workload for the oracle: the workload's first
    sequence lengths (drawn on the host with the workload's recipe) until at least
    min_tokens tokens, all V heads, inputs drawn on the host with the same recipe."""
    from linear_attention_sequence_delta_b200.inputs import WORKLOADS, make_prefill_inputs
    W = dict(WORKLOADS[WORKLOAD])
    g = torch.Generator().manual_seed(seed)
    lens = [int(x) for x in torch.randint(W["len_lo"], W["len_hi"] + 1, (W["num_seqs"],),
                                          generator=g)]
    take = []
    for n in lens:
        take.append(n)
        if sum(take) >= min_tokens:
            break
    for k_ in ("lengths", "num_seqs", "len_lo", "len_hi"):
        W.pop(k_, None)
    return make_prefill_inputs(take, seed=seed, **W)


def _oracle_pass(P):
    """One oracle pass over a whole packed batch (all sequences, all V heads)."""
    import oracle
    t0 = time.perf_counter()
    oracle.forward(P.q, P.k, P.v, P.a, P.b, P.A_log, P.dt_bias,
                   P.cu_seqlens.numpy().astype("int64"), P.initial_state)
    return time.perf_counter() - t0


def cpu_baseline(min_seconds=10.0):
    """The fp64 oracle on this host's cores, on a bounded sample of the headline
    workload (its first sequences, all V heads), repeated for about min_seconds."""
    import oracle
    P = _reference_sample()
    T, H_v = P.q.shape[0], P.v.shape[1]
    reps, total = 0, 0.0
    while total < min_seconds and reps < 60:
        total += _oracle_pass(P)
        reps += 1
    return {"value": reps * T / total, "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{WORKLOAD}: first {P.num_seqs} sequences ({T} tokens), all {H_v} V "
                      f"heads, {reps} passes ({total:.1f} s)"}


def run_reference(args):
    """The oracle (a plain sequential fp64 CPU program) as the reference arm: each step
    is one pass over a bounded sample of the headline workload (its first sequences,
    all V heads), timed as it runs."""
    ws, rank, _ = _dist()
    if rank != 0:
        return
    import oracle
    P = _reference_sample()
    T, H_v = P.q.shape[0], P.v.shape[1]
    for _ in range(args.warmup):
        _oracle_pass(P)
    secs = [_oracle_pass(P) for _ in range(args.steps)]
    ms = 1e3 * sum(secs) / len(secs)
    v = T / (ms / 1e3)
    sample = (f"{WORKLOAD}: first {P.num_seqs} sequences ({T} tokens), all {H_v} V heads, "
              "one pass per step")
    line = {
        "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": WORKLOAD_DESC + "; bf16 q/k/v upcast exactly, fp64 arithmetic",
                   "global_batch": P.num_seqs, "seq_len": T,
                   "parallelism": "host cores (OpenMP over (sequence, V head) units)"},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "kind": "oracle",
                         "cores": oracle.num_threads(), "sample": sample},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--decode-seqs", type=int, default=256,
                    help="sequences per decode step (256 = the decode workload; smaller values "
                         "only for profiling captures)")
    ap.add_argument("--seqs", type=int, default=None,
                    help="sequences of the headline workload (default: its own 64; smaller "
                         "values only for profiling captures)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-mixer", action="store_true",
                    help="skip the conv1d / gated-norm measurements")
    ap.add_argument("--mixer-iters", type=int, default=20)
    ap.add_argument("--no-other-prefill", action="store_true",
                    help="skip the 35B-A3B layer and 397B-A17B long prefill measurements")
    ap.add_argument("--other-iters", type=int, default=10)
    ap.add_argument("--other-prefill", default=",".join(OTHER_PREFILL),
                    help="comma-separated workloads of the other-prefill block")
    ap.add_argument("--other-prefill-seqs", type=int, default=None,
                    help="sequences per other-prefill workload (default: the workload's "
                         "own; smaller values only for profiling captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
