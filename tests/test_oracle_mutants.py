"""The oracle's pins must catch plausible mistakes.

Each case below compiles a copy of the oracle's C source with one planted slip
(on the CPU, into a temporary directory), points the oracle module at it, and
checks that at least one pin in test_oracle_pins fails. The real oracle is put
back afterwards.
"""
import ctypes
import os
import shutil
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")
MIXER_SRC = os.path.join(os.path.dirname(oracle.__file__), "mixer_oracle.c")

MUTANTS = {
    # the P5 reading: read with the undecayed state (decay applied after)
    "decay_after_read": (
        "                /* decay */\n                for (size_t e = 0; e < ssz; ++e) S[e] *= alpha;\n",
        "",
        "                /* write */\n",
        "                for (size_t e = 0; e < ssz; ++e) S[e] *= alpha;\n                /* write */\n",
    ),
    "head_map_modulo": ("const int32_t j = h / r;", "const int32_t j = h % H_qk;", None, None),
    "dropped_beta": ("delta[i] = bt * (vt[i] - kv);", "delta[i] = (vt[i] - kv);", None, None),
    "transposed_read": ("kv += S[(size_t)i * d_k + c] * kn[c];",
                        "kv += S[(size_t)c * d_k + i] * kn[c];", None, None),
    "wrong_delta_sign": ("delta[i] = bt * (vt[i] - kv);", "delta[i] = bt * (vt[i] + kv);",
                         None, None),
    "gate_sign": ("-exp(A_log[h]) * sp", "exp(A_log[h]) * sp", None, None),
    "no_l2norm": ("if (use_l2norm) {", "if (0) {", None, None),
    "readout_before_write": (
        "                /* read-out */\n",
        "",
        None, None),
}

PINS = [
    lambda: pins.test_gates_sign_and_range(),
    lambda: pins.test_gates_closed_forms(),
    *[(lambda a=a: pins.test_brute_force_matrix_form(*a))
      for a in [(3, 1, 2, 3, 2), (4, 2, 4, 4, 3), (4, 1, 3, 2, 4)]],
    lambda: pins.test_brute_force_exact_dyadic(),
    lambda: pins.test_beta_one_unit_key_stores_value(),
    lambda: pins.test_zero_alpha_resets_state(),
    lambda: pins.test_orthogonal_keys_reduce_to_linear_attention(True),
    lambda: pins.test_head_mapping_is_repeat_interleave(),
    lambda: pins.test_l2norm_makes_qk_scale_free(),
]


def _mutate(src, name):
    a, b, c, d = MUTANTS[name]
    if name == "readout_before_write":
        # move the read-out block in front of the write
        start = src.index("                /* read-out */")
        end = src.index("            }\n            if (S_final)")
        block = src[start:end]
        src = src[:start] + src[end:]
        w = src.index("                /* write */")
        return src[:w] + block + src[w:]
    assert a in src, name
    src = src.replace(a, b, 1)
    if c is not None:
        assert c in src, name
        src = src.replace(c, d, 1)
    return src


def _run_pins_on(tmp_path, gdn_src, mixer_src, pins_to_run, name):
    cpath = tmp_path / "m.c"
    cpath.write_text(gdn_src)
    mpath = tmp_path / "mx.c"
    mpath.write_text(mixer_src)
    so = tmp_path / "libm.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", str(cpath), str(mpath),
                           "-o", str(so), "-lm"])
    saved_lib, saved_path = oracle._lib, oracle._LIB_PATH
    try:
        oracle._lib = None
        oracle._LIB_PATH = str(so)
        # keep build() from recompiling the real source over the mutant
        real_build = oracle.build
        oracle.build = lambda force=False: str(so)
        caught = 0
        for pin in pins_to_run:
            try:
                pin()
            except AssertionError:
                caught += 1
        assert caught > 0, f"no pin caught the {name} mutant"
    finally:
        oracle.build = real_build
        oracle._lib, oracle._LIB_PATH = saved_lib, saved_path


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    _run_pins_on(tmp_path, _mutate(open(SRC).read(), name), open(MIXER_SRC).read(), PINS, name)


# planted slips in the convolution / gated-RMSNorm oracle, against its own pins
MIXER_MUTANTS = {
    "conv_taps_reversed": ("acc += w[(int64_t)c * K + i] * XAT(t - (K - 1) + i);",
                           "acc += w[(int64_t)c * K + (K - 1 - i)] * XAT(t - (K - 1) + i);"),
    "conv_window_off_by_one": ("acc += w[(int64_t)c * K + i] * XAT(t - (K - 1) + i);",
                               "acc += w[(int64_t)c * K + i] * XAT(t - K + i);"),
    "conv_cache_newest_first": ("state_in[((int64_t)n * W + (W + (p))) * C + c]",
                                "state_in[((int64_t)n * W + (-1 - (p))) * C + c]"),
    "conv_no_activation": ("y[(s0 + t) * C + c] = oracle_silu(acc);",
                           "y[(s0 + t) * C + c] = acc;"),
    "rms_sum_not_mean": ("const double inv = 1.0 / sqrt(ss / d + eps);",
                         "const double inv = 1.0 / sqrt(ss + eps);"),
    "rms_gate_sigmoid": ("y[r * d + e] = o[r * d + e] * inv * w[e] * oracle_silu(z[r * d + e]);",
                         "y[r * d + e] = o[r * d + e] * inv * w[e] / (1.0 + exp(-z[r * d + e]));"),
}


@pytest.mark.parametrize("name", sorted(MIXER_MUTANTS))
def test_mixer_pins_catch_mutant(name, tmp_path):
    from tests import test_mixer_oracle_pins as mp
    a, b = MIXER_MUTANTS[name]
    src = open(MIXER_SRC).read()
    assert a in src, name
    mixer_pins = [getattr(mp, f) for f in dir(mp) if f.startswith("test_")]
    _run_pins_on(tmp_path, open(SRC).read(), src.replace(a, b, 1), mixer_pins, name)
