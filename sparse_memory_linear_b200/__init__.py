"""B200-native Sparse Delta Memory (SDM) memory pass.

Python binding of libsdm.so, whose C ABI is declared in include/sdm.h.  The binding only
marshals arguments (shapes, data pointers and the current CUDA stream of torch tensors)
and allocates outputs with torch; every step of the pass runs in the sm_100a kernels
behind the ABI.  There is no fallback: if the library is missing the calls raise.
"""

from ._binding import (  # noqa: F401
    ACT,
    ENGINE,
    OPTION,
    ROW_FORMAT,
    SDM_BF16,
    SDM_F32,
    SdmError,
    SdmShape,
    library,
    library_path,
    sdm_decode_step,
    sdm_decode_step_chained,
    sdm_decode_step_coupled,
    sdm_decode_step_coupled_chained,
    sdm_get_device_status,
    sdm_get_option,
    sdm_launch_count,
    sdm_norm_gate,
    sdm_profile_enable,
    sdm_profile_read,
    sdm_scan_forward,
    sdm_scan_forward_coupled,
    sdm_scan_forward_logged,
    sdm_scan_forward_noalloc,
    sdm_select,
    sdm_set_option,
    sdm_slot_cta_stats,
    sdm_state_init,
    sdm_state_pack,
    sdm_state_rows_bytes,
    sdm_state_undo,
    sdm_state_unpack,
    sdm_status_string,
    sdm_undo_workspace_size,
    sdm_workspace_size,
    shape_of,
)
