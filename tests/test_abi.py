"""The C-ABI library on the CPU: it builds, loads, exports every symbol the
header declares, and its host-side validation rejects bad arguments before
touching a device (no compute calls here)."""
import ctypes
import os
import re
import subprocess

import pytest

import sequence_depth_attention_moda_b200 as moda
from sequence_depth_attention_moda_b200 import build as moda_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moda.h")


@pytest.fixture(scope="module")
def lib():
    moda_build.build()
    return moda.load()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moda_[a-z_]+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert header_functions() == sorted(moda.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", moda.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(moda_\w+)", out))
    for name in header_functions():
        assert name in exported, f"{name} declared in moda.h but not exported"
        assert hasattr(lib, name)


def test_status_strings(lib):
    names = [moda.moda_status_string(i) for i in range(7)]
    assert names == ["MODA_OK", "MODA_ERR_INVALID_ARG", "MODA_ERR_MISALIGNED",
                     "MODA_ERR_UNSUPPORTED", "MODA_ERR_WORKSPACE", "MODA_ERR_CUDA",
                     "MODA_ERR_TIMEOUT"]
    assert moda.moda_version() >= 100


def call_fwd(lib, sh, ptrs):
    return lib.moda_fwd(ctypes.byref(sh), *ptrs, None, 0, None)


FAKE = 0x10000   # aligned fake device address: never dereferenced (validation fails first)


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=6, Hk=4), 1),                                         # Hq % Hk
    (dict(d=96), 3),                                                     # bf16 d
    (dict(Hq=256, Hk=1), 3),                                             # G > 128
    (dict(T=-1), 1),
    (dict(L=-2), 1),
    (dict(dtype=7), 1),
    (dict(depth_layout=1, C=0), 1),                                      # chunked needs C
    (dict(depth_layout=1, C=48), 1),                                     # T % C
    (dict(flags=2), 1),                                                  # unknown flag
    (dict(depth_window=3), 1),                                           # window > L
    (dict(depth_window=-1), 1),
    (dict(depth_layout=3), 1),                                           # unknown layout
    (dict(depth_layout=2, L=3), 3),                                      # layer-major: 128 % 3
    (dict(depth_layout=2, L=24), 3),                                     # layer-major: 64 % 24
    (dict(depth_layout=2, L=2, dtype=1), 3),                             # layer-major needs bf16
])
def test_fwd_rejects_bad_shapes(lib, kw, status):
    base = dict(B=1, Hq=4, Hk=2, T=64, d=128, L=2, C=16)
    base.update(kw)
    sh = moda.make_shape(**base)
    rc = call_fwd(lib, sh, [FAKE] * 7)
    assert rc == status, (rc, moda.moda_last_error_message())
    assert moda.moda_last_error_message()


def test_fwd_rejects_null_and_misaligned(lib):
    sh = moda.make_shape(1, 4, 2, 64, 128, 2, 16)
    assert call_fwd(lib, sh, [FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE]) == 1
    assert "V" in moda.moda_last_error_message()
    assert call_fwd(lib, sh, [FAKE, FAKE + 2, FAKE, FAKE, FAKE, FAKE, FAKE]) == 2
    assert call_fwd(lib, sh, [FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE]) == 1   # Kd with L > 0


def test_bwd_rejects_small_workspace(lib):
    sh = moda.make_shape(1, 4, 2, 64, 128, 2, 16)
    need = lib.moda_workspace_size(ctypes.byref(sh), 2)
    assert need == 4 * 4 * 64  # fp32 D = rowsum(dO * O), [B, Hq, T], 256-byte rounded
    rc = lib.moda_bwd(ctypes.byref(sh), *([FAKE] * 13), FAKE, need - 1, None)
    assert rc == 4
    rc = lib.moda_bwd(ctypes.byref(sh), *([FAKE] * 13), None, need, None)
    assert rc == 4


def ws(lib, sh, mode):
    return lib.moda_workspace_size(ctypes.byref(sh), mode)


def test_workspace_sizes(lib):
    sh = moda.make_shape(2, 16, 4, 4096, 128, 16, 64)
    d_rows = 2 * 16 * 4096 * 4                     # D: one fp32 per query row
    # stored dS: one 16 KB tile per (b, hk, 128-row query tile of G=4 heads x
    # 32 tokens, 64-key block)
    tiles = 2 * 4 * (4096 // 32) * (4096 // 64)
    assert ws(lib, sh, 0) == 0
    assert ws(lib, sh, 2) == d_rows
    assert ws(lib, sh, 1) == d_rows + tiles * 16384
    # ragged T: whole tiles, D rounded up to 256 bytes
    sh = moda.make_shape(1, 8, 1, 1000, 128, 3, 0)  # G = 8: 16 tokens per query tile
    assert ws(lib, sh, 2) == (8 * 1000 * 4 + 255) // 256 * 256
    assert ws(lib, sh, 1) == ws(lib, sh, 2) + (-(-1000 // 16)) * (-(-1000 // 64)) * 16384
    # no stored dS: G not in {1, 2, 4, 8}, d = 64, fp32, or more than 16 GiB of tiles
    for s in (moda.make_shape(1, 6, 2, 300, 128, 2, 0), moda.make_shape(1, 4, 2, 300, 64, 2, 0),
              moda.make_shape(1, 4, 2, 300, 128, 2, 0, moda.MODA_FP32),
              moda.make_shape(1, 16, 4, 65536, 128, 32, 64)):
        assert ws(lib, s, 1) == ws(lib, s, 2) > 0
    bad = moda.make_shape(2, 16, 5, 4096, 128, 16, 64)
    assert ws(lib, bad, 1) == ctypes.c_size_t(-1).value
    assert ws(lib, moda.make_shape(1, 4, 2, 64, 128, 2, 0), 3) == ctypes.c_size_t(-1).value


def test_empty_problems_are_noops(lib):
    # B = 0 or T = 0: valid, nothing queued, NULL pointers allowed
    for kw in (dict(B=0), dict(T=0)):
        base = dict(B=1, Hq=4, Hk=2, T=64, d=128, L=2, C=16)
        base.update(kw)
        sh = moda.make_shape(**base)
        assert call_fwd(lib, sh, [None] * 7) == 0
        assert lib.moda_repack_depth(ctypes.byref(sh), None, None, None) == 0


def test_phase_events_validation(lib):
    # n outside 0..8 or a NULL array with n > 0 is rejected; n = 0 turns them off
    assert lib.moda_set_phase_events(None, 0) == 0
    assert lib.moda_set_phase_events(None, 2) == 1
    arr = (ctypes.c_void_p * 9)()
    assert lib.moda_set_phase_events(arr, 9) == 1
    assert lib.moda_set_phase_events(arr, 0) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(T=0), 1),                                                      # no cached key
    (dict(d=96, dtype=moda.MODA_FP32), 3),                               # decode d
    (dict(Hq=64, Hk=2), 3),                                              # G > 16
    (dict(depth_window=5), 1),
])
def test_decode_rejects_bad_shapes(lib, kw, status):
    base = dict(B=1, Hq=4, Hk=2, T=64, d=128, L=2, C=0)
    base.update(kw)
    sh = moda.make_shape(**base)
    rc = lib.moda_decode(ctypes.byref(sh), *([FAKE] * 7), FAKE, 1 << 20, None)
    assert rc == status, (rc, moda.moda_last_error_message())
    assert lib.moda_decode_workspace_size(ctypes.byref(sh)) == ctypes.c_size_t(-1).value


def test_decode_rejects_null_and_empty_batch(lib):
    sh = moda.make_shape(1, 4, 2, 64, 128, 2, 0)
    rc = lib.moda_decode(ctypes.byref(sh), None, *([FAKE] * 6), FAKE, 1 << 20, None)
    assert rc == 1 and "q" in moda.moda_last_error_message()
    sh0 = moda.make_shape(0, 4, 2, 64, 128, 2, 0)
    assert lib.moda_decode(ctypes.byref(sh0), *([None] * 7), None, 0, None) == 0
    assert moda.moda_decode_workspace_size(sh0) == 0


def _decode_ranges_maxc(B, Hk, T, L, window, sms):
    """Independent count of how many CTAs can share one KV head's items when
    n items (per KV head: ceil(rows/64) depth tiles, then ceil(T/64) sequence
    tiles) are cut into `sms` contiguous ranges of floor-divided bounds."""
    rows = L - (L - window if 0 < window < L else 0)
    per = -(-rows // 64) + -(-T // 64)
    n = B * Hk * per
    P = min(n, sms)
    bounds = [c * n // P for c in range(P + 1)]
    worst = 1
    for bh in range(B * Hk):
        first, last = bh * per, (bh + 1) * per - 1
        ctas = [c for c in range(P) if bounds[c] <= last and bounds[c + 1] > first]
        assert ctas == list(range(ctas[0], ctas[-1] + 1))
        worst = max(worst, len(ctas))
    return worst


@pytest.mark.parametrize("B,Hq,Hk,T,d,L,window,dtype", [
    (8, 32, 8, 32768, 128, 48, 0, moda.MODA_BF16),   # the decoding workload
    (3, 16, 2, 4097, 128, 16, 4, moda.MODA_BF16),    # window; CTAs span KV heads
    (64, 16, 8, 200, 64, 4, 0, moda.MODA_BF16),      # many KV heads per CTA
    (1, 4, 4, 1, 64, 3, 0, moda.MODA_BF16),          # fewer items than SMs
    (2, 8, 2, 1000, 128, 8, 0, moda.MODA_FP32),      # fp32: fixed splits
])
def test_decode_workspace_size(lib, B, Hq, Hk, T, d, L, window, dtype):
    """Workspace = one (m, l, o[d]) fp32 record per query head, per CTA that
    can share its KV head's items, per consumer warp (bf16); fp32: per split
    (>= 256 keys each, about 4 CTAs per SM) plus the depth split, per warp.
    Without a GPU the library assumes a 148-SM B200."""
    sh = moda.make_shape(B, Hq, Hk, T, d, L, 0, dtype, depth_window=window)
    got = lib.moda_decode_workspace_size(ctypes.byref(sh))
    if dtype == moda.MODA_BF16:
        parts = _decode_ranges_maxc(B, Hk, T, L, window, 148) * 3
    else:
        want = -(-4 * 148 // (B * Hk))
        splits = max(1, min(want, -(-T // 256)))
        parts = (splits + (1 if L > 0 else 0)) * 8
    need = B * Hq * parts * (d + 2) * 4
    assert got == -(-need // 256) * 256, (got, need)


def test_binding_rejects_host_tensors(lib):
    """A host tensor would hand the kernels a host address: the binding
    refuses it before calling the library."""
    import torch
    sh = moda.make_shape(1, 4, 2, 64, 128, 2, 0)
    q = torch.zeros(1, 4, 64, 128, dtype=torch.bfloat16)
    with pytest.raises(moda.MoDAError) as err:
        moda.moda_fwd(sh, q, None, None, None, None, None, None)
    assert err.value.status == moda.MODA_ERR_INVALID_ARG and "cpu" in str(err.value)
    with pytest.raises(moda.MoDAError):
        moda.moda_decode(sh, torch.zeros(1, 4, 128), *([None] * 6), None, 0)


def test_binding_rejects_wrong_dtype_and_short_tensors(lib):
    """A tensor of the wrong dtype, or with fewer elements than the shape
    implies, would let the kernels read or write past its end: the binding
    refuses it before calling the library (checked before the device check,
    so host tensors show it here)."""
    import torch
    sh = moda.make_shape(1, 4, 2, 64, 128, 2, 0)
    bf = dict(dtype=torch.bfloat16)
    Q, K = torch.zeros(1, 4, 64, 128, **bf), torch.zeros(1, 2, 64, 128, **bf)
    Kd = torch.zeros(1, 2, 128, 128, **bf)
    LSE = torch.zeros(1, 4, 64)
    cases = [
        (dict(Q=Q.float()), "Q has dtype"),
        (dict(Kd=Kd[:, :, :100]), "Kd holds"),
        (dict(LSE=LSE.to(torch.bfloat16)), "LSE has dtype"),
        (dict(LSE=LSE[:, :, :10]), "LSE holds"),
    ]
    for over, msg in cases:
        a = dict(Q=Q, K=K, V=K, Kd=Kd, Vd=Kd, O=Q, LSE=LSE)
        a.update(over)
        with pytest.raises(moda.MoDAError) as err:
            moda.moda_fwd(sh, a["Q"], a["K"], a["V"], a["Kd"], a["Vd"], a["O"], a["LSE"])
        assert err.value.status == moda.MODA_ERR_INVALID_ARG and msg in str(err.value), str(err.value)
    # backward: a short dVd; decoding: a short o; repack: a short destination
    with pytest.raises(moda.MoDAError, match="dVd holds"):
        moda.moda_bwd(sh, Q, K, K, Kd, Kd, Q, LSE, Q, Q, K, K, Kd, Kd[:, :1], None, 0)
    with pytest.raises(moda.MoDAError, match="o holds"):
        moda.moda_decode(sh, torch.zeros(1, 4, 128, **bf), K, K, torch.zeros(1, 2, 2, 128, **bf),
                         torch.zeros(1, 2, 2, 128, **bf), torch.zeros(1, 4, 64, **bf),
                         torch.zeros(1, 4), None, 0)
    with pytest.raises(moda.MoDAError, match="dst holds"):
        moda.moda_repack_depth(sh, torch.zeros(2, 1, 2, 64, 128, **bf), Kd[:, :1])


def test_layer_layout_limits(lib):
    """The layer-major depth layout is accepted exactly when the forward's
    128-row and the dQ kernel's 64-row depth blocks hold whole tokens; the
    decoding and repack entry points ignore the layout field."""
    def ok(**kw):
        base = dict(B=1, Hq=4, Hk=2, T=64, d=128, L=2, C=0, depth_layout=moda.MODA_DEPTH_LAYER)
        base.update(kw)
        sh = moda.make_shape(**base)
        return lib.moda_workspace_size(ctypes.byref(sh), 1) != ctypes.c_size_t(-1).value
    for L in (1, 2, 4, 8, 16, 32, 64):
        assert ok(L=L), L
    assert ok(L=0, dtype=moda.MODA_FP32)                 # no depth rows: nothing to read
    assert not ok(L=48) and not ok(L=3) and not ok(L=128)
    # G = 8: 16 tokens per query tile, blocks of min(c, 16 L rounded to 16) rows
    assert ok(Hq=16, Hk=2, L=3)                          # 48-row blocks: 16 tokens of 3
    assert not ok(Hq=16, Hk=2, L=5)                      # 80 rows: 64-row dQ blocks, 64 % 5
    assert not ok(Hq=16, Hk=2, L=6)                      # 96 rows: 64-row dQ blocks, 64 % 6
    sh = moda.make_shape(B=1, Hq=4, Hk=2, T=64, d=128, L=3, C=0, depth_layout=moda.MODA_DEPTH_LAYER)
    assert lib.moda_decode_workspace_size(ctypes.byref(sh)) != ctypes.c_size_t(-1).value
