"""KDA (Kimi Delta Attention) layer core for NVIDIA B200 (sm_100a).

The compute lives in ``libkda.so`` (CUDA, built from ``csrc/`` by
``gated_delta_rule_152_b200.build``); :mod:`gated_delta_rule_152_b200.kda`
is its ctypes binding.  :mod:`gated_delta_rule_152_b200.inputs` draws the
seeded synthetic workloads.
"""
from .kda import (  # noqa: F401
    KdaError,
    kda_chunk_fwd,
    kda_chunk_fwd_noalloc,
    kda_chunk_fwd_slots,
    kda_chunk_fwd_workspace_size,
    kda_chunk_fwd_workspace_size_min,
    kda_decode_step,
    kda_decode_step_slots,
    kda_selftest_bounded_waits,
    kda_status_string,
    kda_topk_indices,
    kda_topk_workspace_size,
    kda_verify_fwd,
    kda_workspace_error,
    load_library,
)
