"""B200-native Gated DeltaNet decode step.

The work runs in ``libgdn.so`` (hand-written CUDA for sm_100a behind the C ABI of
``include/gdn.h``); this package only marshals torch tensors into that ABI.
"""
from ._abi import (GDN_DEVICE_ERR_SEQLEN, GDN_DEVICE_ERR_SLOT_RANGE, GDN_DEVICE_ERR_TIMEOUT, GDN_ERR_CUDA, GDN_ERR_INVALID_ARGUMENT, GDN_ERR_MISALIGNED,
                   GDN_ERR_SLOT_RANGE, GDN_ERR_UNSUPPORTED, GDN_OK, LIB_PATH, DecodePlan, GdnConfig, GdnError,
                   abi_version, decode_static_scratch_bytes, decode_workspace, decode_workspace_bytes,
                   gdn_decode_step_static_scratch, gdn_decode_step_varlen, gdn_spec_commit, gdn_spec_verify,
                   gdn_in_proj, gdn_out_proj, gdn_decode_step_device_batch, GDN_DEVICE_ERR_BATCH,
                   gdn_selftest_wait_timeout,
                   gdn_check_slots_host, gdn_conv_update, gdn_decode_step, gdn_gated_rmsnorm, gdn_recurrent_step,
                   lib, status_string)

__all__ = [
    "GdnConfig", "GdnError", "DecodePlan", "LIB_PATH", "lib", "status_string", "abi_version",
    "decode_workspace", "decode_workspace_bytes", "gdn_decode_step_static_scratch", "gdn_decode_step_varlen",
    "decode_static_scratch_bytes", "gdn_spec_verify", "gdn_spec_commit", "gdn_in_proj", "gdn_out_proj", "gdn_decode_step_device_batch", "GDN_DEVICE_ERR_BATCH",
    "gdn_selftest_wait_timeout",
    "gdn_conv_update", "gdn_recurrent_step", "gdn_gated_rmsnorm", "gdn_decode_step", "gdn_check_slots_host",
    "GDN_OK", "GDN_ERR_INVALID_ARGUMENT", "GDN_ERR_UNSUPPORTED", "GDN_ERR_MISALIGNED", "GDN_ERR_SLOT_RANGE",
    "GDN_ERR_CUDA", "GDN_DEVICE_ERR_SLOT_RANGE", "GDN_DEVICE_ERR_TIMEOUT", "GDN_DEVICE_ERR_SEQLEN",
]
