"""B200-native speculative verification: Python binding of ``libsv.so``.

Argument marshalling only: every step of the verification path runs in the
library's CUDA kernels (see ``include/sv.h``).  PyTorch supplies device
memory and streams.  There is no CPU fallback: if the library cannot be
loaded, every call raises.
"""
from ._binding import (  # noqa: F401
    SV_BF16, SV_F32, SV_NOTE_CDF_FALLBACK, SV_NOTE_ZERO_RESIDUAL, SV_ROW_BAD_LENGTH,
    SV_ROW_BAD_TEMPERATURE, SV_ROW_BAD_TOKEN, SVError, lib, library_path, sv_philox4x32_10,
    sv_debug_sts_timeouts, sv_debug_sts_wait_limit, sv_philox_uniforms, sv_profile_begin,
    sv_profile_read, sv_schedule, sv_schedule_admit, sv_schedule_verify,
    sv_status_string, sv_sts_apply, sv_sts_fit, sv_sts_workspace_bytes,
    sv_verify, sv_verify_debug, sv_verify_host, sv_verify_host_workspace_bytes, sv_verify_launches,
    sv_verify_noalloc, sv_verify_workspace_bytes,
    sv_vp_decide, sv_vp_draw, sv_vp_slice, sv_vp_stats, sv_vp_stats_bytes, sv_vp_workspace_bytes,
    verify, vp_slice,
)
