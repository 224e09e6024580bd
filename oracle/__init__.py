"""CPU fp64 oracle for the fused MoDA attention operator.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  The product path (the
CUDA library and its Python binding) never imports it, and it imports nothing
from the product package.

The arithmetic lives in ``moda_oracle.c`` (plain C, double precision, OpenMP
over independent rows); this module only builds that file with gcc and
marshals numpy arrays through ctypes.  See the C file's header for the
definitions it follows:

* "Mixture-of-Depths Attention" paper summary (arXiv 2603.15619), section
  "Mixture-of-Depths Attention (MoDA): The Unified Operator": the joint-softmax
  equation with its sequence causal mask and depth matching mask.
* "moda-attention 0.1.0" PyPI page, "Using the Kernel Directly" (tensor
  layouts) and "Key Design Choices" (GQA by repeat_interleave).
* Paper summary, "Hardware-Efficient Implementation" (layer-major versus
  token-major depth layout, for the repack).

``decode`` evaluates the newest token's rows through the same C row function.

Parity status: the forward, backward and repack are pinned by the CPU tests
(the pins live in ``tests/oracle_pins.py`` and run from ``tests/test_oracle.py``):
library special cases, closed forms, invariants, an independent dense brute
force, autograd, finite differences and an exact worked example
(``tests/golden/``); ``tests/test_oracle_mutants.py`` checks that planted
mistakes fail them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moda_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libmoda_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no GPU needed).  Returns the .so path."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", _SRC,
                           "-o", tmp, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load_library(path: str | None = None):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if path is None and _lib is not None:
        return _lib
    with _lock:
        lib = ctypes.CDLL(path or build())
        i, d = ctypes.c_int, ctypes.c_double
        lib.moda_oracle_fwd.argtypes = [i, i, i, i, i, i, d] + [_dp] * 7
        lib.moda_oracle_fwd.restype = i
        lib.moda_oracle_fwd_ex.argtypes = [i, i, i, i, i, i, d, i, i] + [_dp] * 7
        lib.moda_oracle_fwd_ex.restype = i
        lib.moda_oracle_bwd.argtypes = [i, i, i, i, i, i, d] + [_dp] * 11
        lib.moda_oracle_bwd.restype = i
        lib.moda_oracle_bwd_ex.argtypes = [i, i, i, i, i, i, d, i, i] + [_dp] * 11
        lib.moda_oracle_bwd_ex.restype = i
        lib.moda_oracle_row.argtypes = [i, i, i, d] + [_dp] * 8
        lib.moda_oracle_row.restype = None
        lib.moda_oracle_repack.argtypes = [i, i, i, i, i, i, ctypes.c_void_p, ctypes.c_void_p]
        lib.moda_oracle_repack.restype = i
        lib.moda_oracle_threads.argtypes = []
        lib.moda_oracle_threads.restype = i
        if path is None:
            _lib = lib
        return lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor on the CPU
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a: np.ndarray | None):
    if a is None:
        return ctypes.cast(0, _dp)
    return a.ctypes.data_as(_dp)


def _shape(Q, K, Kd):
    B, Hq, T, d = Q.shape
    Hk = K.shape[1]
    assert K.shape == (B, Hk, T, d), (K.shape, Q.shape)
    L = 0 if Kd is None else Kd.shape[2] // max(T, 1)
    if Kd is not None:
        assert Kd.shape == (B, Hk, T * L, d), (Kd.shape, Q.shape, K.shape)
    return B, Hq, Hk, T, d, L


def threads(lib=None) -> int:
    """OpenMP threads the oracle's parallel loops use."""
    return int((lib or load_library()).moda_oracle_threads())


def fwd(Q, K, V, Kd=None, Vd=None, scale: float = 0.0, lib=None, causal: bool = True,
        window: int = 0):
    """Forward: returns (O [B,Hq,T,d], LSE [B,Hq,T]) in float64.

    Kd/Vd are the token-major depth tensors [B,Hk,T*L,d]; pass None (or
    empty arrays) for L = 0.  scale <= 0 selects 1/sqrt(d).  causal=False
    drops the sequence mask; window > 0 keeps each token's last `window`
    depth rows only.
    """
    lib = lib or load_library()
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    Kd = None if Kd is None or np.size(Kd) == 0 else _f64(Kd)
    Vd = None if Vd is None or np.size(Vd) == 0 else _f64(Vd)
    B, Hq, Hk, T, d, L = _shape(Q, K, Kd)
    O = np.zeros((B, Hq, T, d))
    LSE = np.zeros((B, Hq, T))
    rc = lib.moda_oracle_fwd_ex(B, Hq, Hk, T, d, L, float(scale), int(bool(causal)), int(window),
                                _ptr(Q), _ptr(K), _ptr(V), _ptr(Kd), _ptr(Vd), _ptr(O), _ptr(LSE))
    if rc != 0:
        raise ValueError("oracle rejected the shape")
    return O, LSE


def bwd(Q, K, V, Kd, Vd, dO, scale: float = 0.0, lib=None, causal: bool = True, window: int = 0):
    """Backward: returns (dQ, dK, dV, dKd, dVd) in float64 (same options as fwd)."""
    lib = lib or load_library()
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    Kd = None if Kd is None or np.size(Kd) == 0 else _f64(Kd)
    Vd = None if Vd is None or np.size(Vd) == 0 else _f64(Vd)
    B, Hq, Hk, T, d, L = _shape(Q, K, Kd)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    dKd = np.zeros((B, Hk, T * L, d))
    dVd = np.zeros((B, Hk, T * L, d))
    rc = lib.moda_oracle_bwd_ex(B, Hq, Hk, T, d, L, float(scale), int(bool(causal)), int(window),
                                _ptr(Q), _ptr(K), _ptr(V), _ptr(Kd), _ptr(Vd), _ptr(dO), _ptr(dQ),
                                _ptr(dK), _ptr(dV), _ptr(dKd if L else None),
                                _ptr(dVd if L else None))
    if rc != 0:
        raise ValueError("oracle rejected the shape")
    return dQ, dK, dV, dKd, dVd


def row(q, Kseq, Vseq, Kdep, Vdep, scale: float = 0.0, lib=None, return_p: bool = False):
    """One query row: one softmax over exactly the given visible rows.

    q [d]; Kseq/Vseq [n_seq, d] (for the causal operator at token t, the KV
    head's rows 0..t); Kdep/Vdep [n_dep, d] (token t's visible depth rows).
    Returns (o [d], lse) or (o, lse, p) where p is the normalised
    [seq | depth] weight row.
    """
    lib = lib or load_library()
    q, Kseq, Vseq = _f64(q), _f64(Kseq), _f64(Vseq)
    Kdep, Vdep = _f64(Kdep), _f64(Vdep)
    d = q.shape[-1]
    n_seq = Kseq.shape[0]
    L = Kdep.shape[0]
    if scale <= 0:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros(d)
    lse = np.zeros(1)
    p = np.zeros(n_seq + L) if return_p else None
    lib.moda_oracle_row(n_seq, L, d, float(scale), _ptr(q), _ptr(Kseq), _ptr(Vseq),
                        _ptr(Kdep if L else None), _ptr(Vdep if L else None),
                        _ptr(o), _ptr(lse), _ptr(p))
    return (o, float(lse[0]), p) if return_p else (o, float(lse[0]))


def decode(q, K, V, Kd=None, Vd=None, window: int = 0, scale: float = 0.0, lib=None):
    """Decoding: the newest token's query rows against T cached keys and its
    own L depth rows -- one row of the operator per (b, h) (the causal mask
    admits every cached key).  q [B,Hq,d]; K, V [B,Hk,T,d]; Kd, Vd [B,Hk,L,d]
    or None; window > 0 keeps the last `window` depth rows.  Returns
    (o [B,Hq,d], lse [B,Hq]) in float64."""
    lib = lib or load_library()
    q, K, V = _f64(q), _f64(K), _f64(V)
    B, Hq, d = q.shape
    Hk = K.shape[1]
    G = Hq // Hk
    L = 0 if Kd is None or np.size(Kd) == 0 else Kd.shape[2]
    Kd = _f64(Kd) if L else np.zeros((B, Hk, 0, d))
    Vd = _f64(Vd) if L else np.zeros((B, Hk, 0, d))
    lo = L - window if 0 < window < L else 0
    o = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            o[b, h], lse[b, h] = row(q[b, h], K[b, hk], V[b, hk], Kd[b, hk, lo:], Vd[b, hk, lo:],
                                     scale=scale, lib=lib)
    return o, lse


def repack(src, B: int, Hk: int, T: int, d: int, L: int, lib=None) -> np.ndarray:
    """Layer-major [L,B,Hk,T,d] -> token-major [B,Hk,T*L,d]; bytewise copy."""
    lib = lib or load_library()
    src = np.ascontiguousarray(src)
    assert src.shape == (L, B, Hk, T, d), src.shape
    dst = np.empty((B, Hk, T * L, d), dtype=src.dtype)
    rc = lib.moda_oracle_repack(B, Hk, T, d, L, src.dtype.itemsize,
                                src.ctypes.data_as(ctypes.c_void_p),
                                dst.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError("oracle rejected the shape")
    return dst
