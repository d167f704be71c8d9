"""B200-native (sm_100a) selective state-space scan of Mamba.

The work runs in libssmscan.so (hand-written CUDA kernels behind a C ABI,
declared in include/ssm_scan.h); this package is a thin ctypes binding with
the same entry-point names. PyTorch supplies device memory and streams.
"""
from ._binding import (  # noqa: F401
    SSM_DTYPE_BF16,
    SSM_DTYPE_F32,
    ScanPlan,
    SsmError,
    conv1d_silu_bwd_workspace_bytes,
    lib,
    scan_bwd_workspace_bytes,
    scan_plan,
    scan_workspace_bytes,
    ssm_compose_carries,
    ssm_conv1d_silu_bwd,
    ssm_conv1d_silu_fwd,
    ssm_conv1d_silu_update,
    ssm_delta_sum,
    ssm_scan_bwd,
    ssm_scan_fwd,
    ssm_scan_fwd_noalloc,
    ssm_scan_status,
    ssm_scan_status_noalloc,
    ssm_ssd_scan_fwd,
    ssm_ssd_scan_status,
    ssm_ssd_state_update,
    ssm_state_update,
)

__all__ = ["ssm_scan_fwd", "ssm_scan_fwd_noalloc", "ssm_scan_bwd", "ssm_state_update",
           "ssm_scan_status", "ssm_scan_status_noalloc", "scan_plan", "scan_workspace_bytes", "scan_bwd_workspace_bytes",
           "ssm_conv1d_silu_fwd", "ssm_conv1d_silu_bwd", "ssm_conv1d_silu_update",
           "conv1d_silu_bwd_workspace_bytes",
           "ssm_delta_sum", "ssm_compose_carries", "ssm_ssd_scan_fwd", "ssm_ssd_scan_status",
           "ssm_ssd_state_update",
           "SsmError", "ScanPlan", "SSM_DTYPE_F32", "SSM_DTYPE_BF16", "lib"]
