"""Gated DeltaNet token mixer on NVIDIA B200 (sm_100a).

The compute lives in libgdn.so (CUDA kernels behind the C ABI of
include/gdn.h); `gdn` is its ctypes binding and `inputs` draws seeded
synthetic inputs of the Qwen3.5 GDN layer shapes.
"""
from .gdn import (GDNError, gdn_conv1d_silu, gdn_conv1d_silu_decode,  # noqa: F401
                  gdn_decode_slots, gdn_decode_step, gdn_decode_step_bf16_state, gdn_gates,
                  gdn_mixer_prefill, gdn_prefill, gdn_prefill_slots, gdn_rmsnorm_gated,
                  gdn_sync_status, load_library, mixer_workspace_size, workspace_size)
