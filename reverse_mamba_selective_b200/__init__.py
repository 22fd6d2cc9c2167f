"""B200-native right-to-left selective-scan sidecar (R2LM) and partial-bidirectional scan.

The compute lives in libr2l.so (CUDA, sm_100a; C ABI in include/r2l.h).  This
package only builds it (``_build``) and marshals arguments to it (``r2l``).
"""

from .r2l import (  # noqa: F401
    R2L_BF16, R2L_ERR_CUDA, R2L_ERR_INVALID_ARG, R2L_ERR_TIMEOUT, R2L_ERR_UNSUPPORTED, R2L_F32, R2L_OK,
    R2LError, ScanArgs, SidecarWeights, bidir_scan, fwd_scan_from_state, load, make_scan_args, make_sidecar_weights,
    r2l_abi_version, r2l_decode_step, r2l_device_status, r2l_dt_proj, r2l_in_proj, r2l_residual_apply, r2l_scan_block,
    r2l_scan_block_bwd,
    r2l_sidecar_forward, r2l_wait_selftest, r2l_x_proj, r2l_x_proj_noalloc, sidecar_workspace_size, status_string,
)
