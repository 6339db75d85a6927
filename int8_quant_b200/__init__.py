"""B200-native (sm_100a) Mamba-2 SSD chunked scan: bf16 and W8A8 (persistent INT8 state).

The compute lives in libssd.so (hand-written CUDA); `ssd` is its ctypes binding and
`runner` allocates device buffers with torch and sequences the calls.
"""
from .ssd import (SsdShape, SsdI8Params, SsdError, library, shape_of, i8_params,  # noqa: F401
                  SSD_STORAGE_ACS_FP16, SSD_STORAGE_CB_INT8,
                  ssd_workspace_bytes, ssd_calibrate_workspace_bytes, ssd_quantize_inputs,
                  ssd_scan_fwd_bf16, ssd_scan_fwd_bf16_static, ssd_static_scratch_status, ssd_scan_fwd_i8, ssd_scan_fwd_i8_debug, ssd_calibrate_i8,
                  ssd_workspace_status, ssd_profile_enable, ssd_profile_read, ssd_profile_reset, ssd_profile_filter,
                  ssd_selftest_bounded_wait, ssd_scan_fwd_bf16_from_state, ssd_scan_fwd_i8_from_state,
                  ssd_decode_step_bf16, ssd_decode_step_i8, ssd_out_proj_workspace_bytes, ssd_out_proj_i8,
                  ssd_out_proj_status)
