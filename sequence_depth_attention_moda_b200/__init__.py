"""B200-native fused Mixture-of-Depths Attention (MoDA) operator.

The compute lives in ``lib/libmoda.so`` (hand-written CUDA for sm_100a behind
the C ABI of ``include/moda.h``); ``_binding`` marshals torch tensors into it
and ``ops`` offers tensor-allocating conveniences over the same entry points.
"""
from ._binding import (EXPORTED, LIB_PATH, MODA_BF16, MODA_DEPTH_CHUNKED, MODA_DEPTH_FLAT,
                       MODA_FP32, MoDAError, load, make_shape, moda_bwd, moda_bwd_noalloc,
                       moda_check_status, moda_fwd, moda_last_error_message, moda_repack_depth, moda_set_phase_events,
                       moda_shape, moda_status_string, moda_version, moda_workspace_size)

__all__ = ["EXPORTED", "LIB_PATH", "MODA_BF16", "MODA_DEPTH_CHUNKED", "MODA_DEPTH_FLAT",
           "MODA_FP32", "MoDAError", "load", "make_shape", "moda_bwd", "moda_bwd_noalloc", "moda_check_status",
           "moda_fwd", "moda_last_error_message", "moda_repack_depth", "moda_set_phase_events", "moda_shape",
           "moda_status_string", "moda_version", "moda_workspace_size"]
