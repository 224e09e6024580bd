"""Decoding on the GPU against the oracle: one new token per sequence over T
cached keys plus its own depth rows (the newest row of the operator).
Every output row is checked, including at the full decode workload."""
import numpy as np
import pytest
import torch

import oracle
import sequence_depth_attention_moda_b200 as moda
from sequence_depth_attention_moda_b200 import inputs as I
from moda_cases import BF16_MAX_ABS, BF16_MEAN_ABS, FP32_MAX_ABS, LSE_MAX_ABS, Guarded, err_stats, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    yield
    moda.moda_check_status()


def run_decode(w, x):
    sh = moda.make_shape(w.B, w.Hq, w.Hk, w.T, w.d, w.L, 0,
                         moda.MODA_BF16 if w.dtype == "bf16" else moda.MODA_FP32,
                         depth_window=w.window)
    nws = moda.moda_decode_workspace_size(sh)
    ws = torch.empty(max(nws, 16), device=DEV, dtype=torch.uint8)
    gd = Guarded()
    o = gd.like("o", x["q"])
    lse = gd.empty("lse", (w.B, w.Hq), torch.float32, DEV)
    moda.moda_decode(sh, x["q"], x["K"], x["V"], x["Kd"] if w.L else None, x["Vd"] if w.L else None,
                     o, lse, ws, nws)
    gd.check()
    return o, lse


def check(w, x, o, lse):
    ref_o, ref_lse = oracle.decode(f64(x["q"]), f64(x["K"]), f64(x["V"]),
                                   f64(x["Kd"]) if w.L else None, f64(x["Vd"]) if w.L else None,
                                   window=w.window)
    mx, mean = err_stats(f64(o), ref_o)
    assert np.all(np.isfinite(f64(o)))
    if w.dtype == "fp32":
        assert mx <= FP32_MAX_ABS, mx
    else:
        assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS, (mx, mean)
    assert err_stats(f64(lse), ref_lse)[0] <= LSE_MAX_ABS


CASES = [  # B, Hq, Hk, d, T, L, window, dtype
    (2, 8, 2, 128, 1000, 8, 0, "bf16"),
    (1, 4, 4, 64, 1, 3, 0, "bf16"),        # only the token's own key
    (3, 16, 2, 128, 4097, 16, 4, "bf16"),  # G = 8, depth window
    (1, 16, 1, 128, 777, 0, 0, "bf16"),    # G = 16, no depth
    (2, 6, 2, 128, 300, 6, 0, "bf16"),     # G = 3
    (1, 4, 2, 64, 500, 5, 2, "fp32"),
    (1, 2, 2, 128, 33, 40, 0, "fp32"),     # more depth rows than keys per warp tile
    (2, 8, 2, 128, 65, 100, 0, "bf16"),    # two depth tiles; last sequence tile holds one key
    (1, 4, 1, 128, 64, 100, 70, "bf16"),   # depth window starting inside a tile
    (1, 2, 1, 64, 63, 64, 0, "bf16"),      # one key short of a tile, exactly one depth tile
    (64, 16, 8, 64, 200, 4, 0, "bf16"),    # many KV heads per CTA range, ring wraps
    (2, 32, 8, 128, 4096, 48, 0, "bf16"),  # d = 128: the ring wraps (7 items per CTA)
    (8, 8, 8, 128, 100, 0, 0, "bf16"),     # G = 1, no depth
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%d_Hq%d_Hk%d_d%d_T%d_L%d_S%d_%s" % c)
def test_decode_small(case):
    B, Hq, Hk, d, T, L, window, dtype = case
    w = I.Workload("dec", B=B, Hq=Hq, Hk=Hk, d=d, T=T, L=L, C=0, dtype=dtype, seed=77, window=window)
    x = I.make_decode_inputs(w, device=DEV)
    o, lse = run_decode(w, x)
    check(w, x, o, lse)


def test_decode_full_workload():
    w = I.DECODE_T32K
    x = I.make_decode_inputs(w, device=DEV)
    o, lse = run_decode(w, x)
    check(w, x, o, lse)


def test_decode_deterministic():
    w = I.DECODE_T32K.with_(T=5000)
    x = I.make_decode_inputs(w, device=DEV)
    o1, l1 = run_decode(w, x)
    o2, l2 = run_decode(w, x)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_decode_workspace_too_small():
    w = I.DECODE_T32K.with_(T=1000)
    x = I.make_decode_inputs(w, device=DEV)
    sh = moda.make_shape(w.B, w.Hq, w.Hk, w.T, w.d, w.L, 0)
    nws = moda.moda_decode_workspace_size(sh)
    ws = torch.empty(nws, device=DEV, dtype=torch.uint8)
    o = torch.empty_like(x["q"])
    lse = torch.empty(w.B, w.Hq, device=DEV, dtype=torch.float32)
    with pytest.raises(moda.MoDAError) as err:
        moda.moda_decode(sh, x["q"], x["K"], x["V"], x["Kd"], x["Vd"], o, lse, ws, nws - 256)
    assert err.value.status == moda.MODA_ERR_WORKSPACE
