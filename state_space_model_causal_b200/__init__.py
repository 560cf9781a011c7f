"""B200-native Mamba hot path: causal conv1d, fused prefill selective scan and
single-token selective_state_update (plus the sequence-piece calls and the
double-gated short conv of an LFM2-style conv block), behind the C-ABI library
``libssm_causal.so`` (declared in ``include/ssm_causal.h``).

The functions below are the thin ctypes binding of the C entry points; they
raise if the library has not been built (there is no fallback path).
"""
from .binding import (LaunchInfo, SsmError, library, ssm_causal_conv1d_fwd,  # noqa: F401
                      ssm_device_error, ssm_device_error_info, ssm_gated_conv1d_fwd,
                      ssm_scan_carry_fold,
                      ssm_scan_delta_sum, ssm_selective_scan_fwd, ssm_selective_scan_fwd_noalloc,
                      ssm_selective_scan_workspace_size, ssm_selective_state_update)
