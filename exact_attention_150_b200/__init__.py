"""Exact scaled-dot-product attention for B200 (sm_100a).

The computation runs in libattn.so (C ABI in include/attn.h); this package
holds its build script, its ctypes binding and the seeded synthetic workloads.
"""

from .native import (AttnError, attn_bwd, attn_bwd_deterministic, attn_bwd_phase, attn_bwd_varlen,
                     attn_bwd_varlen_workspace_bytes, attn_bwd_workspace_bytes, attn_fwd, attn_fwd_fp8,
                     attn_fwd_varlen, attn_host_step, attn_host_step_device_bytes, attn_last_device_status, backward,
                     backward_varlen, device_status, forward, forward_fp8, forward_fp8_varlen, forward_varlen, host_step, load,
                     status_string)

__all__ = ["AttnError", "attn_fwd", "attn_bwd", "attn_bwd_deterministic", "attn_bwd_phase", "attn_bwd_workspace_bytes",
           "attn_last_device_status", "forward", "backward", "device_status", "load", "status_string",
           "attn_fwd_varlen", "attn_bwd_varlen", "attn_bwd_varlen_workspace_bytes", "forward_varlen",
           "backward_varlen", "attn_fwd_fp8", "forward_fp8", "attn_host_step", "attn_host_step_device_bytes",
           "host_step", "attn_fwd_fp8_varlen", "forward_fp8_varlen"]
