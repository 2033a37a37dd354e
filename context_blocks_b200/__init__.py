"""Blockwise (ring-step) attention for NVIDIA B200, as a C-ABI CUDA library.

``attn_fwd`` attends every query row to one K/V chunk and returns the
normalised partial output with its natural log-sum-exp; ``attn_merge``
combines partial results over disjoint chunks into the exact full result;
``blockwise_attention`` chains the two over a list of chunks.  The kernels
live in ``libpa_attn.so`` (``include/pa_attn.h``); this package only loads it
and marshals arguments.  Build it with ``python -m context_blocks_b200.build``.
"""

from ._binding import (LIB_PATH, PA_ACCUM_FINAL, PA_ACCUM_FIRST, PA_ERR_BAD_INPUT, PA_ERR_CUDA, PA_ERR_INVALID_ARG,
                       PA_ERR_MISALIGNED, PA_ERR_TIMEOUT, PA_ERR_UNSUPPORTED, PA_OK, PaError, attn_chunks_noalloc,
                       attn_fwd, attn_fwd_accum, attn_fwd_chunks, attn_fwd_fp8, attn_merge, last_error, load_library,
                       poll_device_status, quantize_e4m3, residual_diff, selftest_timeout, set_wait_limit_ms,
                       status_string, version)
from .ring import blockwise_attention

__all__ = ["LIB_PATH", "PA_OK", "PA_ERR_INVALID_ARG", "PA_ERR_UNSUPPORTED", "PA_ERR_MISALIGNED",
           "PA_ERR_CUDA", "PA_ERR_TIMEOUT", "PA_ERR_BAD_INPUT", "PA_ACCUM_FIRST", "PA_ACCUM_FINAL", "PaError",
           "attn_chunks_noalloc", "attn_fwd", "attn_fwd_accum", "attn_fwd_chunks", "attn_fwd_fp8", "attn_merge",
           "blockwise_attention", "last_error", "load_library", "poll_device_status", "quantize_e4m3", "residual_diff",
           "selftest_timeout", "set_wait_limit_ms", "status_string", "version"]
