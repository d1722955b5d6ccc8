"""Gated-retention (gRet) mixer on NVIDIA B200: Python face of libgret.

The mixer ("YOCO 深度技术分析", section 2.2; chunkwise form, section 5.3.2)
runs entirely in the CUDA library ``libgret.so`` built from ``csrc/``; this
package only marshals arguments (see ``gret.py``).
"""
from .gret import (  # noqa: F401
    Dtype, Epilogue, GretError, LIB_PATH, Path, SIGNATURES, Status, check_device_status, decode_step,
    gret_decode_step, gret_last_device_status, gret_prefill, gret_prefill_backward,
    gret_prefill_backward_launches, gret_prefill_backward_workspace_size, gret_prefill_from_state,
    gret_prefill_launches,
    gret_prefill_noalloc, gret_prefill_path, gret_prefill_state, gret_prefill_state_workspace_size,
    gret_prefill_varlen, gret_prefill_workspace_size, gret_state_fold,
    gret_set_profile_events, gret_status_string, gret_version, load, prefill, prefill_backward, prefill_path, prefill_state,
    prefill_varlen, state_fold, prefill_projected, gret_prefill_projected, gret_prefill_projected_workspace_size,
    gret_prefill_resume, gret_debug_inject_timeout, gret_set_gate_profile_events,
    gret_prefill_varlen_workspace_size, gret_prefill_varlen_launches,
)
