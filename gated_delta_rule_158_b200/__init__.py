"""libkda: Kimi Delta Attention (KDA) kernels for B200 (sm_100a).

The compute lives in the C-ABI library libkda.so (include/kda.h; its
KDA_DEBUG_CHECKS build with device-side bounds checks is libkda_debug.so,
selected with select_library(debug=True)); this package is its thin ctypes
binding plus the seeded workload generators.
Build the library with ``python -m gated_delta_rule_158_b200.build``.
"""
from ._lib import (  # noqa: F401
    KDA_BF16, KDA_ERR_BAD_SEQLENS, KDA_ERR_BOUNDS, KDA_ERR_CUDA, KDA_ERR_INVALID_ARG,
    KDA_ERR_MISALIGNED, KDA_ERR_TIMEOUT, KDA_ERR_UNSUPPORTED, KDA_ERR_WORKSPACE, KDA_F32, KDA_OK, KdaError,
    kda_chunk_fwd, kda_chunk_fwd_gated, kda_chunk_fwd_gated_host,
    kda_chunk_fwd_gated_host_workspace_size, kda_chunk_fwd_noalloc, kda_chunk_fwd_workspace_size,
    kda_chunk_segment_transition, kda_chunk_state_prefix, kda_debug_checks_enabled,
    kda_decode_step,
    kda_decode_replay, kda_decode_step_gated, kda_decode_verify, kda_gate_bwd,
    kda_gate_bwd_workspace_size, kda_gate_fwd,
    kda_get_device_status, kda_last_cuda_error_string, kda_noalloc_get_device_status, kda_recurrent_bwd,
    kda_recurrent_bwd_workspace_size, kda_selftest_bounded_wait, kda_selftest_bounds_check,
    kda_set_wait_limit_ns, kda_status_string,
    lib, select_library)
