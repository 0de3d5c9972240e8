"""Exact IO-aware attention (forward and backward) for B200 / sm_100a.

The computation lives in the CUDA library ``libfa_b200.so`` (C ABI in
``include/fa.h``); this package is its ctypes binding.  ``workloads`` names the
synthetic workloads and draws their seeded inputs.
"""

from .binding import (  # noqa: F401
    FA_BF16, FA_FP16, FA_OK, FA_ERR_CUDA, FA_ERR_INVALID_ARG, FA_ERR_MISALIGNED,
    FA_ERR_TIMEOUT, FA_ERR_UNSUPPORTED, FaError, attention_bwd, attention_decode_paged,
    attention_fwd, attention_fwd_fp8, fa_bwd, fa_decode_paged, fa_fwd_fp8, fa_decode_workspace_bytes,
    fa_bwd_dropout, fa_bwd_window, fa_bwd_workspace_bytes, fa_fwd, fa_fwd_dropout,
    fa_fwd_window, fa_get_device_status, fa_peek_device_status_word,
    fa_selftest_wait_timeout, fa_set_bwd_max_blocks, fa_set_profile_events, fa_status_string, fa_bwd_noalloc, load,
    KERNEL_FWD, KERNEL_BWD_MAIN,
)
