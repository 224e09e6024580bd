"""B200-native fused Mixture-of-Depths Attention (MoDA) operator.

The compute lives in ``lib/libmoda.so`` (hand-written CUDA for sm_100a behind
the C ABI of ``include/moda.h``); ``_binding`` marshals torch tensors into it,
with the same names as the C entry points.  ``inputs`` draws the seeded
synthetic workloads; ``build`` compiles the library.
"""
from ._binding import (
    EXPORTED, LIB_PATH, MODA_BF16, MODA_DEPTH_CHUNKED, MODA_DEPTH_FLAT, MODA_DEPTH_LAYER,
    MODA_ERR_CUDA, MODA_ERR_INVALID_ARG, MODA_ERR_MISALIGNED, MODA_ERR_TIMEOUT, MODA_ERR_UNSUPPORTED,
    MODA_ERR_WORKSPACE, MODA_FLAG_NONCAUSAL, MODA_FP32, MODA_OK, MoDAError, load, make_shape,
    moda_bwd, moda_bwd_noalloc, moda_check_status, moda_decode, moda_decode_workspace_size,
    moda_fwd, moda_last_error_message, moda_repack_depth, moda_selftest_wait_timeout,
    moda_set_phase_events, moda_shape, moda_status_string, moda_version, moda_workspace_size)

__all__ = [
    "EXPORTED", "LIB_PATH", "MODA_BF16", "MODA_DEPTH_CHUNKED", "MODA_DEPTH_FLAT", "MODA_DEPTH_LAYER",
    "MODA_ERR_CUDA",
    "MODA_ERR_INVALID_ARG", "MODA_ERR_MISALIGNED", "MODA_ERR_TIMEOUT", "MODA_ERR_UNSUPPORTED",
    "MODA_ERR_WORKSPACE", "MODA_FLAG_NONCAUSAL", "MODA_FP32", "MODA_OK", "MoDAError", "load",
    "make_shape", "moda_bwd", "moda_bwd_noalloc", "moda_check_status", "moda_decode",
    "moda_decode_workspace_size", "moda_fwd", "moda_last_error_message", "moda_repack_depth",
    "moda_selftest_wait_timeout", "moda_set_phase_events", "moda_shape", "moda_status_string",
    "moda_version", "moda_workspace_size"]
