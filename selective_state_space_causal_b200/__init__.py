"""B200-native (sm_100a) selective-SSM mixer core.

The computation lives in ``libssm_causal.so`` (hand-written CUDA behind the C
ABI declared in ``include/ssm_causal.h``); this package is its thin Python
binding. Importing it loads the library and fails loudly if it is missing.
"""

from ._lib import (  # noqa: F401
    SSM_BF16,
    SSM_F32,
    SsmError,
    lib,
    replay_buffers,
    ssm_causal_conv1d,
    ssm_conv_scan_fwd,
    ssm_check_cu_seqlens,
    ssm_last_error,
    ssm_launch_count,
    ssm_probe_rate,
    ssm_probe_sink_floats,
    ssm_device_status,
    ssm_replay_flush,
    ssm_replay_reset,
    ssm_replay_state_update,
    ssm_scan_bwd_workspace_size,
    ssm_scan_workspace_size,
    ssm_selective_scan_bwd,
    ssm_selective_scan_fwd,
    ssm_selective_scan_fwd_ckpt,
    ssm_selective_scan_fwd_noalloc,
    ssm_selective_state_update,
    ssm_selftest_wait_timeout,
    ssm_scan_bwd_variant_for,
    ssm_scan_variant_for,
    ssm_set_scan_bwd_variant,
    ssm_set_scan_variant,
    ssm_version,
)
