"""ctypes binding of libmoda (include/moda.h): argument marshalling only.

Every function here has the name of the C entry point it wraps and takes
torch tensors (or raw integer device pointers) plus an optional stream.  No
arithmetic of the operator happens in Python; if the shared library is
missing the first call raises, there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libmoda.so")

MODA_OK = 0
MODA_ERR_INVALID_ARG = 1
MODA_ERR_MISALIGNED = 2
MODA_ERR_UNSUPPORTED = 3
MODA_ERR_WORKSPACE = 4
MODA_ERR_CUDA = 5
MODA_ERR_TIMEOUT = 6

MODA_BF16 = 0
MODA_FP32 = 1
MODA_DEPTH_FLAT = 0
MODA_DEPTH_CHUNKED = 1
MODA_DEPTH_LAYER = 2
MODA_FLAG_NONCAUSAL = 1

# Every symbol include/moda.h declares.
EXPORTED = ("moda_workspace_size", "moda_repack_depth", "moda_fwd", "moda_bwd",
            "moda_bwd_noalloc", "moda_decode", "moda_decode_workspace_size",
            "moda_set_phase_events", "moda_check_status",
            "moda_selftest_wait_timeout", "moda_status_string", "moda_last_error_message",
            "moda_version")


class moda_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hk", ctypes.c_int),
                ("T", ctypes.c_int), ("d", ctypes.c_int), ("L", ctypes.c_int),
                ("C", ctypes.c_int), ("dtype", ctypes.c_int), ("depth_layout", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("flags", ctypes.c_int),
                ("depth_window", ctypes.c_int)]


class MoDAError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {status_name(status)} ({detail})")


_lock = threading.Lock()
_lib = None


def load(path: Optional[str] = None):
    """Load libmoda.so.  Raises if it has not been built (no fallback)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"libmoda.so not found at {p}; build it with "
                               "`python -m sequence_depth_attention_moda_b200.build`")
        lib = ctypes.CDLL(p)
        vp, sz, i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        sp = ctypes.POINTER(moda_shape)
        lib.moda_workspace_size.argtypes = [sp, i]
        lib.moda_workspace_size.restype = sz
        lib.moda_repack_depth.argtypes = [sp, vp, vp, vp]
        lib.moda_repack_depth.restype = i
        lib.moda_fwd.argtypes = [sp] + [vp] * 7 + [vp, sz, vp]
        lib.moda_fwd.restype = i
        lib.moda_bwd.argtypes = [sp] + [vp] * 13 + [vp, sz, vp]
        lib.moda_bwd.restype = i
        lib.moda_bwd_noalloc.argtypes = [sp] + [vp] * 13 + [vp]
        lib.moda_bwd_noalloc.restype = i
        lib.moda_decode_workspace_size.argtypes = [sp]
        lib.moda_decode_workspace_size.restype = sz
        lib.moda_decode.argtypes = [sp] + [vp] * 7 + [vp, sz, vp]
        lib.moda_decode.restype = i
        lib.moda_set_phase_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), i]
        lib.moda_set_phase_events.restype = i
        lib.moda_check_status.argtypes = [vp]
        lib.moda_check_status.restype = i
        lib.moda_selftest_wait_timeout.argtypes = [vp]
        lib.moda_selftest_wait_timeout.restype = i
        lib.moda_status_string.argtypes = [i]
        lib.moda_status_string.restype = ctypes.c_char_p
        lib.moda_last_error_message.argtypes = []
        lib.moda_last_error_message.restype = ctypes.c_char_p
        lib.moda_version.argtypes = []
        lib.moda_version.restype = i
        if path is None:
            _lib = lib
        return lib


def status_name(status: int) -> str:
    try:
        return load().moda_status_string(status).decode()
    except Exception:  # library missing: still give a readable name
        return f"status {status}"


def make_shape(B, Hq, Hk, T, d, L, C=0, dtype=MODA_BF16, depth_layout=MODA_DEPTH_FLAT,
               softmax_scale=0.0, flags=0, depth_window=0) -> moda_shape:
    return moda_shape(int(B), int(Hq), int(Hk), int(T), int(d), int(L), int(C), int(dtype),
                      int(depth_layout), float(softmax_scale), int(flags), int(depth_window))


def _ptr(x) -> Optional[int]:
    """Device address of a buffer argument: None, a raw int address (passed
    through), or a tensor that must be contiguous and on the current CUDA
    device (the kernels read row-major device memory; a host or strided
    tensor is rejected here rather than read wrongly)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_cuda:
        raise MoDAError(MODA_ERR_INVALID_ARG, "argument", f"tensor on {x.device}, not a CUDA device")
    if not x.is_contiguous():
        raise MoDAError(MODA_ERR_INVALID_ARG, "argument", "tensor is not contiguous (row-major)")
    import torch
    if x.device.index != torch.cuda.current_device():
        raise MoDAError(MODA_ERR_INVALID_ARG, "argument",
                        f"tensor on {x.device}, current device is cuda:{torch.cuda.current_device()}")
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _expect(where: str, shape: moda_shape, specs):
    """Check tensor arguments against the shape before the C call: each spec
    is (name, tensor or int or None, element count, "io" or "f32").  A tensor
    must hold at least that many elements of the shape's dtype ("io") or of
    float32 ("f32"); raw integer addresses and None pass through (the library
    checks NULL itself)."""
    import torch
    io = torch.bfloat16 if shape.dtype == MODA_BF16 else torch.float32
    for name, x, count, kind in specs:
        if x is None or isinstance(x, int):
            continue
        want = torch.float32 if kind == "f32" else io
        if x.dtype != want:
            raise MoDAError(MODA_ERR_INVALID_ARG, where, f"{name} has dtype {x.dtype}, expected {want}")
        if x.numel() < count:
            raise MoDAError(MODA_ERR_INVALID_ARG, where,
                            f"{name} holds {x.numel()} elements, the shape needs {count}")


def _sizes(shape: moda_shape):
    B, Hq, Hk, T, d, L = (max(0, int(v)) for v in (shape.B, shape.Hq, shape.Hk, shape.T, shape.d,
                                                   shape.L))
    return {"q": B * Hq * T * d, "kv": B * Hk * T * d, "dep": B * Hk * T * L * d, "lse": B * Hq * T}


def _check(rc: int, where: str):
    if rc != MODA_OK:
        detail = load().moda_last_error_message().decode()
        raise MoDAError(rc, where, detail)


def moda_workspace_size(shape: moda_shape, for_bwd) -> int:
    """for_bwd: 0/False forward, 1/True backward at its fastest, 2 the least
    the backward accepts."""
    n = load().moda_workspace_size(ctypes.byref(shape), int(for_bwd))
    if n == ctypes.c_size_t(-1).value:
        _check(load().moda_fwd(ctypes.byref(shape), *([None] * 7), None, 0, None), "moda_workspace_size")
    return int(n)


def moda_repack_depth(shape: moda_shape, src, dst, stream=None):
    n = _sizes(shape)["dep"]
    _expect("moda_repack_depth", shape, [("src", src, n, "io"), ("dst", dst, n, "io")])
    _check(load().moda_repack_depth(ctypes.byref(shape), _ptr(src), _ptr(dst), _stream(stream)),
           "moda_repack_depth")


def moda_fwd(shape: moda_shape, Q, K, V, Kd, Vd, O, LSE, ws=None, ws_bytes: int = 0, stream=None):
    n = _sizes(shape)
    _expect("moda_fwd", shape, [("Q", Q, n["q"], "io"), ("K", K, n["kv"], "io"), ("V", V, n["kv"], "io"),
                                ("Kd", Kd, n["dep"], "io"), ("Vd", Vd, n["dep"], "io"),
                                ("O", O, n["q"], "io"), ("LSE", LSE, n["lse"], "f32")])
    _check(load().moda_fwd(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(Kd), _ptr(Vd),
                           _ptr(O), _ptr(LSE), _ptr(ws), int(ws_bytes), _stream(stream)), "moda_fwd")


def _bwd_specs(shape, Q, K, V, Kd, Vd, O, LSE, dO, dQ, dK, dV, dKd, dVd):
    n = _sizes(shape)
    return [("Q", Q, n["q"], "io"), ("K", K, n["kv"], "io"), ("V", V, n["kv"], "io"),
            ("Kd", Kd, n["dep"], "io"), ("Vd", Vd, n["dep"], "io"), ("O", O, n["q"], "io"),
            ("LSE", LSE, n["lse"], "f32"), ("dO", dO, n["q"], "io"), ("dQ", dQ, n["q"], "io"),
            ("dK", dK, n["kv"], "io"), ("dV", dV, n["kv"], "io"), ("dKd", dKd, n["dep"], "io"),
            ("dVd", dVd, n["dep"], "io")]


def _check_ws(where: str, ws, ws_bytes: int):
    """A workspace tensor must hold the ws_bytes the call claims."""
    if ws is None or isinstance(ws, int):
        return
    have = ws.numel() * ws.element_size()
    if have < int(ws_bytes):
        raise MoDAError(MODA_ERR_INVALID_ARG, where, f"ws holds {have} bytes, ws_bytes says {int(ws_bytes)}")


def moda_bwd(shape: moda_shape, Q, K, V, Kd, Vd, O, LSE, dO, dQ, dK, dV, dKd, dVd, ws,
             ws_bytes: int, stream=None):
    _expect("moda_bwd", shape, _bwd_specs(shape, Q, K, V, Kd, Vd, O, LSE, dO, dQ, dK, dV, dKd, dVd))
    _check_ws("moda_bwd", ws, ws_bytes)
    _check(load().moda_bwd(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(Kd), _ptr(Vd),
                           _ptr(O), _ptr(LSE), _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dKd),
                           _ptr(dVd), _ptr(ws), int(ws_bytes), _stream(stream)), "moda_bwd")


def moda_bwd_noalloc(shape: moda_shape, Q, K, V, Kd, Vd, O, LSE, dO, dQ, dK, dV, dKd, dVd,
                     stream=None):
    """moda_bwd for callers that cannot allocate: no workspace argument; the
    library's built-in scratch holds at most B*Hq*T = 4,194,304 query rows,
    and overlapping calls on the GPU share (and race on) that scratch."""
    _expect("moda_bwd_noalloc", shape, _bwd_specs(shape, Q, K, V, Kd, Vd, O, LSE, dO, dQ, dK, dV, dKd,
                                                  dVd))
    _check(load().moda_bwd_noalloc(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(Kd),
                                   _ptr(Vd), _ptr(O), _ptr(LSE), _ptr(dO), _ptr(dQ), _ptr(dK),
                                   _ptr(dV), _ptr(dKd), _ptr(dVd), _stream(stream)),
           "moda_bwd_noalloc")


def moda_set_phase_events(events) -> None:
    """Timing markers: `events` is a list of torch.cuda.Event (or raw
    cudaEvent_t ints) the following moda_fwd / moda_bwd calls of this thread
    record between their kernel launches; [] turns them off."""
    handles = [e if isinstance(e, int) else e.cuda_event for e in events]
    arr = (ctypes.c_void_p * max(1, len(handles)))(*handles)
    _check(load().moda_set_phase_events(arr, len(handles)), "moda_set_phase_events")


def moda_check_status(stream=None):
    _check(load().moda_check_status(_stream(stream)), "moda_check_status")


def moda_decode_workspace_size(shape: moda_shape) -> int:
    n = load().moda_decode_workspace_size(ctypes.byref(shape))
    if n == ctypes.c_size_t(-1).value:   # report the validation error itself
        _check(load().moda_decode(ctypes.byref(shape), *([None] * 7), None, 0, None),
               "moda_decode_workspace_size")
    return int(n)


def moda_decode(shape: moda_shape, q, K, V, Kd, Vd, o, lse, ws, ws_bytes: int, stream=None):
    B, Hq, Hk, T, d, L = (max(0, int(v)) for v in (shape.B, shape.Hq, shape.Hk, shape.T, shape.d,
                                                   shape.L))
    _expect("moda_decode", shape, [("q", q, B * Hq * d, "io"), ("K", K, B * Hk * T * d, "io"),
                                   ("V", V, B * Hk * T * d, "io"), ("Kd", Kd, B * Hk * L * d, "io"),
                                   ("Vd", Vd, B * Hk * L * d, "io"), ("o", o, B * Hq * d, "io"),
                                   ("lse", lse, B * Hq, "f32")])
    _check_ws("moda_decode", ws, ws_bytes)
    _check(load().moda_decode(ctypes.byref(shape), _ptr(q), _ptr(K), _ptr(V), _ptr(Kd), _ptr(Vd),
                              _ptr(o), _ptr(lse), _ptr(ws), int(ws_bytes), _stream(stream)),
           "moda_decode")


def moda_selftest_wait_timeout(stream=None):
    """Queue the bounded-wait self-test; the next moda_check_status raises
    MoDAError with MODA_ERR_TIMEOUT."""
    _check(load().moda_selftest_wait_timeout(_stream(stream)), "moda_selftest_wait_timeout")


def moda_status_string(status: int) -> str:
    return load().moda_status_string(int(status)).decode()


def moda_last_error_message() -> str:
    return load().moda_last_error_message().decode()


def moda_version() -> int:
    return int(load().moda_version())
