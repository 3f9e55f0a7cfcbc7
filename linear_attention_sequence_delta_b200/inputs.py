"""Seeded synthetic inputs for the Gated DeltaNet token mixer.

This module only draws random numbers; it holds none of the method's
arithmetic. The tests, the benchmark and the smoke check all take their inputs
from here, so the CUDA path and the oracle always see the same values.

Recipe (one torch.Generator seeded with `seed`, on the device the tensors are
made on, drawn in this fixed order):
  1. sequence lengths (packed batches only), integers in [len_lo, len_hi];
  2. q, k  [T, H_qk, d_k] and v [T, H_v, d_v] ~ N(0, 1) in fp32, then rounded
     to bf16 (round-to-nearest-even) when the I/O type is bf16;
  3. a, b  [T, H_v] ~ N(0, 1), fp32;
  4. A_log [H_v] ~ U(0, ln 16), dt_bias [H_v] ~ U(-1, 1), fp32;
  5. initial state [N, H_v, d_v, d_k] ~ N(0, state_std^2), fp32 (when asked for).
For the steps around the delta rule (make_mixer_inputs, drawn in this order):
  1. sequence lengths as above;
  2. x [T, C] ~ N(0, 1) (C = conv_dim = 2 H_qk d_k + H_v d_v, the concatenated
     q/k/v channels), rounded to the I/O type;
  3. conv weight [C, K] ~ U(-1/sqrt(K), 1/sqrt(K)), conv bias [C] ~ N(0, 0.1^2)
     (used only where a test asks for a bias), fp32;
  4. conv cache [N, K-1, C] ~ N(0, 1), rounded to the I/O type;
  5. o, z [T, H_v, d_v] ~ N(0, 1), rounded to the I/O type; norm weight
     [d_v] ~ U(0.5, 1.5), fp32.
The shapes follow the Qwen3.5 GDN layers: 16 QK heads, 32 (35B-A3B) or 64
(397B-A17B) V heads, head dim 128. The CPU and CUDA generators produce
different streams; a given test always draws on one device.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import torch


@dataclass
class PrefillInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    a: torch.Tensor
    b: torch.Tensor
    A_log: torch.Tensor
    dt_bias: torch.Tensor
    cu_seqlens: torch.Tensor  # int32 [N+1]
    initial_state: Optional[torch.Tensor]

    @property
    def num_seqs(self) -> int:
        return self.cu_seqlens.numel() - 1

    @property
    def total_tokens(self) -> int:
        return self.q.shape[0]

    def to(self, device) -> "PrefillInputs":
        mv = lambda t: None if t is None else t.to(device)
        return PrefillInputs(*(mv(getattr(self, f)) for f in self.__dataclass_fields__))


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_prefill_inputs(lengths=None, *, num_seqs: int = 1, seq_len: int = 256,
                        len_lo: int = 128, len_hi: int = 8192, H_qk: int = 16,
                        H_v: int = 32, d_k: int = 128, d_v: int = 128,
                        io_dtype: torch.dtype = torch.bfloat16,
                        state_std: Optional[float] = None, seed: int = 0,
                        device="cpu") -> PrefillInputs:
    """Draw one packed batch.

    lengths: None -> num_seqs sequences of seq_len tokens each;
             "random" -> num_seqs lengths drawn uniformly in [len_lo, len_hi];
             a list -> those lengths.
    """
    g = _gen(device, seed)
    if isinstance(lengths, str) and lengths == "random":
        lens = torch.randint(len_lo, len_hi + 1, (num_seqs,), generator=g, device=device)
        lens = [int(x) for x in lens.cpu()]
    elif lengths is None:
        lens = [seq_len] * num_seqs
    else:
        lens = [int(x) for x in lengths]
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    T = cu[-1]
    f32 = torch.float32
    q = torch.randn((T, H_qk, d_k), generator=g, device=device, dtype=f32).to(io_dtype)
    k = torch.randn((T, H_qk, d_k), generator=g, device=device, dtype=f32).to(io_dtype)
    v = torch.randn((T, H_v, d_v), generator=g, device=device, dtype=f32).to(io_dtype)
    a = torch.randn((T, H_v), generator=g, device=device, dtype=f32)
    b = torch.randn((T, H_v), generator=g, device=device, dtype=f32)
    A_log = torch.rand((H_v,), generator=g, device=device, dtype=f32) * math.log(16.0)
    dt_bias = torch.rand((H_v,), generator=g, device=device, dtype=f32) * 2.0 - 1.0
    S0 = None
    if state_std is not None:
        S0 = torch.randn((len(lens), H_v, d_v, d_k), generator=g, device=device,
                         dtype=f32) * state_std
    cu_t = torch.tensor(cu, dtype=torch.int32, device=device)
    return PrefillInputs(q, k, v, a, b, A_log, dt_bias, cu_t, S0)


@dataclass
class DecodeInputs:
    q: torch.Tensor      # [steps, N, H_qk, d_k]
    k: torch.Tensor      # [steps, N, H_qk, d_k]
    v: torch.Tensor      # [steps, N, H_v, d_v]
    a: torch.Tensor      # [steps, N, H_v]
    b: torch.Tensor      # [steps, N, H_v]
    A_log: torch.Tensor  # [H_v]
    dt_bias: torch.Tensor
    state: torch.Tensor  # [N, H_v, d_v, d_k] fp32


def make_decode_inputs(*, steps: int, num_seqs: int = 256, H_qk: int = 16, H_v: int = 64,
                       d_k: int = 128, d_v: int = 128, io_dtype: torch.dtype = torch.bfloat16,
                       state_std: float = 0.02, seed: int = 0, device="cpu") -> DecodeInputs:
    """Draw `steps` consecutive single-token inputs for num_seqs sequences."""
    g = _gen(device, seed)
    f32 = torch.float32
    N = num_seqs
    q = torch.randn((steps, N, H_qk, d_k), generator=g, device=device, dtype=f32).to(io_dtype)
    k = torch.randn((steps, N, H_qk, d_k), generator=g, device=device, dtype=f32).to(io_dtype)
    v = torch.randn((steps, N, H_v, d_v), generator=g, device=device, dtype=f32).to(io_dtype)
    a = torch.randn((steps, N, H_v), generator=g, device=device, dtype=f32)
    b = torch.randn((steps, N, H_v), generator=g, device=device, dtype=f32)
    A_log = torch.rand((H_v,), generator=g, device=device, dtype=f32) * math.log(16.0)
    dt_bias = torch.rand((H_v,), generator=g, device=device, dtype=f32) * 2.0 - 1.0
    state = torch.randn((N, H_v, d_v, d_k), generator=g, device=device, dtype=f32) * state_std
    return DecodeInputs(q, k, v, a, b, A_log, dt_bias, state)


@dataclass
class MixerInputs:
    x: torch.Tensor            # [T, C]
    conv_weight: torch.Tensor  # [C, K] fp32
    conv_bias: torch.Tensor    # [C] fp32
    conv_state: torch.Tensor   # [N, K-1, C]
    o: torch.Tensor            # [T, H_v, d_v]
    z: torch.Tensor            # [T, H_v, d_v]
    norm_weight: torch.Tensor  # [d_v] fp32
    cu_seqlens: torch.Tensor   # int32 [N+1]

    def to(self, device) -> "MixerInputs":
        return MixerInputs(*(getattr(self, f).to(device) for f in self.__dataclass_fields__))


def make_mixer_inputs(lengths=None, *, num_seqs: int = 1, seq_len: int = 256,
                      len_lo: int = 128, len_hi: int = 8192, H_qk: int = 16, H_v: int = 32,
                      d_k: int = 128, d_v: int = 128, kernel_size: int = 4,
                      io_dtype: torch.dtype = torch.bfloat16, seed: int = 0,
                      device="cpu") -> MixerInputs:
    """Inputs of the convolution in front of the delta rule and of the gated norm after it."""
    g = _gen(device, seed)
    if isinstance(lengths, str) and lengths == "random":
        lens = torch.randint(len_lo, len_hi + 1, (num_seqs,), generator=g, device=device)
        lens = [int(x) for x in lens.cpu()]
    elif lengths is None:
        lens = [seq_len] * num_seqs
    else:
        lens = [int(x) for x in lengths]
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    T, N, K = cu[-1], len(lens), kernel_size
    C = 2 * H_qk * d_k + H_v * d_v
    f32 = torch.float32
    x = torch.randn((T, C), generator=g, device=device, dtype=f32).to(io_dtype)
    bound = 1.0 / math.sqrt(K)
    w = (torch.rand((C, K), generator=g, device=device, dtype=f32) * 2.0 - 1.0) * bound
    bias = torch.randn((C,), generator=g, device=device, dtype=f32) * 0.1
    st = torch.randn((N, K - 1, C), generator=g, device=device, dtype=f32).to(io_dtype)
    o = torch.randn((T, H_v, d_v), generator=g, device=device, dtype=f32).to(io_dtype)
    z = torch.randn((T, H_v, d_v), generator=g, device=device, dtype=f32).to(io_dtype)
    nw = torch.rand((d_v,), generator=g, device=device, dtype=f32) + 0.5
    cu_t = torch.tensor(cu, dtype=torch.int32, device=device)
    return MixerInputs(x, w, bias, st, o, z, nw, cu_t)


@dataclass
class MixerPrefillInputs:
    x: torch.Tensor              # [T, C] pre-conv q | k | v channels
    conv_weight: torch.Tensor    # [C, K] fp32
    conv_bias: torch.Tensor      # [C] fp32
    conv_state: torch.Tensor     # [N, K-1, C]
    a: torch.Tensor              # [T, H_v] fp32
    b: torch.Tensor
    A_log: torch.Tensor          # [H_v] fp32
    dt_bias: torch.Tensor
    initial_state: Optional[torch.Tensor]  # [N, H_v, d_v, d_k] fp32
    z: torch.Tensor              # [T, H_v, d_v]
    norm_weight: torch.Tensor    # [d_v] fp32
    cu_seqlens: torch.Tensor     # int32 [N+1]
    H_qk: int

    @property
    def num_seqs(self) -> int:
        return self.cu_seqlens.numel() - 1

    def to(self, device) -> "MixerPrefillInputs":
        mv = lambda t: t.to(device) if isinstance(t, torch.Tensor) else t
        return MixerPrefillInputs(*(mv(getattr(self, f)) for f in self.__dataclass_fields__))


def make_mixer_prefill_inputs(lengths=None, *, num_seqs: int = 1, seq_len: int = 256,
                              len_lo: int = 128, len_hi: int = 8192, H_qk: int = 16,
                              H_v: int = 32, d: int = 128, kernel_size: int = 4,
                              io_dtype: torch.dtype = torch.bfloat16,
                              state_std: Optional[float] = None, seed: int = 0,
                              device="cpu") -> MixerPrefillInputs:
    """Inputs of the whole mixer core (conv -> delta rule -> gated norm), drawn in this
    order: lengths (as make_prefill_inputs); x [T, C] ~ N(0, 1) (C = (2 H_qk + H_v) d,
    rounded to the I/O type); conv weight [C, K] ~ U(-1/sqrt(K), 1/sqrt(K)), conv bias
    [C] ~ N(0, 0.1^2); conv cache [N, K-1, C] ~ N(0, 1) (rounded); a, b [T, H_v] ~ N(0, 1);
    A_log ~ U(0, ln 16), dt_bias ~ U(-1, 1); initial state ~ N(0, state_std^2) (when
    asked for); z [T, H_v, d] ~ N(0, 1) (rounded); norm weight [d] ~ U(0.5, 1.5)."""
    g = _gen(device, seed)
    if isinstance(lengths, str) and lengths == "random":
        lens = torch.randint(len_lo, len_hi + 1, (num_seqs,), generator=g, device=device)
        lens = [int(x) for x in lens.cpu()]
    elif lengths is None:
        lens = [seq_len] * num_seqs
    else:
        lens = [int(x) for x in lengths]
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    T, N, K = cu[-1], len(lens), kernel_size
    C = (2 * H_qk + H_v) * d
    f32 = torch.float32
    x = torch.randn((T, C), generator=g, device=device, dtype=f32).to(io_dtype)
    bound = 1.0 / math.sqrt(K)
    w = (torch.rand((C, K), generator=g, device=device, dtype=f32) * 2.0 - 1.0) * bound
    bias = torch.randn((C,), generator=g, device=device, dtype=f32) * 0.1
    st = torch.randn((N, K - 1, C), generator=g, device=device, dtype=f32).to(io_dtype)
    a = torch.randn((T, H_v), generator=g, device=device, dtype=f32)
    b = torch.randn((T, H_v), generator=g, device=device, dtype=f32)
    A_log = torch.rand((H_v,), generator=g, device=device, dtype=f32) * math.log(16.0)
    dt_bias = torch.rand((H_v,), generator=g, device=device, dtype=f32) * 2.0 - 1.0
    S0 = None
    if state_std is not None:
        S0 = torch.randn((N, H_v, d, d), generator=g, device=device, dtype=f32) * state_std
    z = torch.randn((T, H_v, d), generator=g, device=device, dtype=f32).to(io_dtype)
    nw = torch.rand((d,), generator=g, device=device, dtype=f32) + 0.5
    cu_t = torch.tensor(cu, dtype=torch.int32, device=device)
    return MixerPrefillInputs(x, w, bias, st, a, b, A_log, dt_bias, S0, z, nw, cu_t, H_qk)


# The five workloads, by name. Sizes are those of the Qwen3.5 GDN layers.
WORKLOADS = {
    "tiny_fp32": dict(num_seqs=1, seq_len=256, H_qk=2, H_v=4, d_k=64, d_v=64,
                      io_dtype=torch.float32),
    "prefill_35b": dict(num_seqs=1, seq_len=4096, H_qk=16, H_v=32, d_k=128, d_v=128),
    "prefill_397b_long": dict(num_seqs=4, seq_len=16384, H_qk=16, H_v=64, d_k=128, d_v=128),
    "varlen_64": dict(lengths="random", num_seqs=64, len_lo=128, len_hi=8192, H_qk=16,
                      H_v=32, d_k=128, d_v=128, state_std=0.02),
}
DECODE_WORKLOAD = dict(num_seqs=256, H_qk=16, H_v=64, d_k=128, d_v=128, state_std=0.02)
DECODE_STEPS = 1000
