"""B200-native (sm_100a) selective state-space scan (S6): a C-ABI CUDA library
(libssm_scan.so, declared in include/ssm_scan.h) and its thin Python binding."""
from .binding import (  # noqa: F401
    ConvSpec,
    FwdOptions,
    SsmError,
    load,
    new_workspace,
    selective_scan_bwd,
    selective_scan_fwd,
    ssm_read_status,
    ssm_selective_scan_bwd,
    ssm_selective_scan_bwd_ex,
    ssm_selective_scan_bwd_workspace_size,
    ssm_selective_scan_fwd,
    ssm_selective_scan_fwd_conv,
    ssm_selective_scan_fwd_noalloc,
    ssm_selective_scan_workspace_size,
    ssm_state_update,
    ssm_state_update_conv,
    ssm_workspace_init,
    status_string,
)
