"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle
on the same seeded inputs.

Tolerances (bf16 in / fp32 accumulate): output max-abs <= 2e-2 and mean-abs
<= 2e-3; fp32 path max-abs <= 1e-4; LSE max-abs <= 1e-3; gradients relative
to each reference tensor's own scale, with no floor: normwise <= 1e-2,
max-abs <= 2e-2 * max|ref|, mean-abs <= 5e-3 * mean|ref| (storing a gradient
in bf16 alone costs up to 2^-9 relative).  Small cases are compared element
by element in full; the full-size workloads on sampled rows (forward) and
sampled (b, hk) slices (backward), which the oracle computes exactly for what
they cover.  Every output sits between guard bands and starts as NaN (see
moda_cases.Guarded): writes outside a tensor or elements left unwritten fail.
"""
import numpy as np
import pytest
import torch

import oracle
import sequence_depth_attention_moda_b200 as moda
from sequence_depth_attention_moda_b200 import inputs as I
from moda_cases import (LSE_MAX_ABS, assert_grad_close, assert_out_close, err_stats, f64,
                        oracle_bwd_full, oracle_fwd_full, oracle_rows, run_gpu, sample_rows,
                        slice_workload, token_major)

pytestmark = pytest.mark.gpu

DEV = "cuda"

# (B, Hq, Hk, d, T, L): ragged T, every G the tile handles (incl. G not dividing 128), d in {64,128}
SMALL = [
    (1, 4, 2, 128, 300, 4),
    (2, 8, 2, 64, 257, 3),
    (1, 4, 4, 128, 200, 1),
    (1, 16, 2, 128, 130, 16),
    (1, 6, 2, 128, 100, 5),
    (1, 4, 2, 128, 256, 0),
    (1, 2, 1, 128, 1, 7),
    (1, 32, 1, 64, 64, 2),
    (1, 128, 1, 64, 9, 3),
    (1, 8, 2, 128, 513, 40),
]


def small_w(B, Hq, Hk, d, T, L, seed=2024, backward=False):
    return I.Workload(f"small_{B}_{Hq}_{Hk}_{d}_{T}_{L}", B=B, Hq=Hq, Hk=Hk, d=d, T=T, L=L, C=1,
                      seed=seed, backward=backward)


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    yield
    moda.moda_check_status()


# ------------------------------------------------------------------ repack --
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_repack_bit_exact(dtype):
    w = I.Workload("rp", B=2, Hq=4, Hk=2, d=128 if dtype == "bf16" else 40, T=37, L=5, C=1,
                   dtype=dtype, seed=5)
    x = I.make_inputs(w, device=DEV)
    out = run_gpu(w, x, backward=False)
    Kd_ref, Vd_ref = token_major(x, w)
    assert torch.equal(out["Kd"].cpu(), Kd_ref) and torch.equal(out["Vd"].cpu(), Vd_ref)


def test_repack_bit_exact_full_size():
    w = I.TRAIN_FWD_BWD
    x = I.make_inputs(w, device=DEV, grad_out=False)
    sh = moda.make_shape(w.B, w.Hq, w.Hk, w.T, w.d, w.L, w.C)
    Kd = torch.empty(w.B, w.Hk, w.T * w.L, w.d, device=DEV, dtype=torch.bfloat16)
    moda.moda_repack_depth(sh, x["Kd_layer"], Kd)
    rng = np.random.default_rng(3)
    for _ in range(64):
        b, hk, t, l = (int(rng.integers(n)) for n in (w.B, w.Hk, w.T, w.L))
        assert torch.equal(Kd[b, hk, t * w.L + l], x["Kd_layer"][l, b, hk, t])
    # the whole tensor, bit for bit, against the library's own permute
    ref = x["Kd_layer"].permute(1, 2, 3, 0, 4).reshape(w.B, w.Hk, w.T * w.L, w.d)
    assert torch.equal(Kd, ref)


# ------------------------------------------------------------------ forward -
def test_fwd_fp32_tiny_config():
    w = I.TINY_FP32
    x = I.make_inputs(w, device=DEV)
    out = run_gpu(w, x)
    O, LSE = oracle_fwd_full(w, x)
    assert_out_close(f64(out["O"]), O, "fp32", "O")
    assert err_stats(f64(out["LSE"]), LSE)[0] <= 1e-4


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "B%d_Hq%d_Hk%d_d%d_T%d_L%d" % c)
def test_fwd_bf16_small(case):
    w = small_w(*case)
    x = I.make_inputs(w, device=DEV)
    out = run_gpu(w, x, backward=False)
    O, LSE = oracle_fwd_full(w, x)
    assert_out_close(f64(out["O"]), O, "bf16", "O")
    assert err_stats(f64(out["LSE"]), LSE)[0] <= LSE_MAX_ABS


def test_fwd_qk_scaled_distribution_small():
    w = small_w(2, 16, 4, 128, 700, 16).with_(qk_scaled=True)
    x = I.make_inputs(w, device=DEV)
    out = run_gpu(w, x, backward=False)
    O, LSE = oracle_fwd_full(w, x)
    assert_out_close(f64(out["O"]), O, "bf16", "O")


def _check_rows(w, x, out, n_random=24):
    rows = sample_rows(w, n_random)
    O_ref, LSE_ref = oracle_rows(w, x, out["Kd"], out["Vd"], rows)
    got = np.stack([f64(out["O"][b, h, t]) for (b, h, t) in rows])
    lse = np.array([float(out["LSE"][b, h, t]) for (b, h, t) in rows])
    assert_out_close(got, O_ref, w.dtype, f"{w.name} O rows")
    assert err_stats(lse, LSE_ref)[0] <= LSE_MAX_ABS, f"{w.name} LSE rows"


def test_fwd_layer_T4k_sampled():
    w = I.LAYER_1P5B
    x = I.make_inputs(w, device=DEV)
    _check_rows(w, x, run_gpu(w, x, backward=False))


@pytest.mark.parametrize("L", [32, 0])
def test_fwd_long_context_T64k_sampled(L):
    w = I.LONG_64K.with_(L=L)
    x = I.make_inputs(w, device=DEV)
    _check_rows(w, x, run_gpu(w, x, backward=False), n_random=16)


def test_fwd_depth_group_sweep_sampled():
    for w in I.depth_group_sweep():
        x = I.make_inputs(w, device=DEV)
        _check_rows(w, x, run_gpu(w, x, backward=False, layout=moda.MODA_DEPTH_CHUNKED), n_random=6)
        del x
        torch.cuda.empty_cache()


def test_fwd_train_shape_sampled():
    w = I.TRAIN_FWD_BWD
    x = I.make_inputs(w, device=DEV, grad_out=False)
    _check_rows(w, x, run_gpu(w, x, backward=False))


def test_fwd_bitwise_identical_across_layouts_and_C():
    w = small_w(1, 16, 4, 128, 1024, 8)
    x = I.make_inputs(w, device=DEV)
    ref = run_gpu(w, x, backward=False)
    for C in (32, 64, 128, 1024):
        o = run_gpu(w, x, backward=False, layout=moda.MODA_DEPTH_CHUNKED, C=C)
        assert torch.equal(o["O"], ref["O"]) and torch.equal(o["LSE"], ref["LSE"])


def test_fwd_deterministic():
    w = small_w(2, 8, 2, 128, 777, 9)
    x = I.make_inputs(w, device=DEV)
    a = run_gpu(w, x, backward=False)
    b = run_gpu(w, x, backward=False)
    assert torch.equal(a["O"], b["O"]) and torch.equal(a["LSE"], b["LSE"])


# ----------------------------------------------------------------- backward -
BWD_SMALL = [c for c in SMALL if c[4] > 1] + [(1, 4, 2, 128, 1, 3)]


@pytest.mark.parametrize("case", BWD_SMALL, ids=lambda c: "B%d_Hq%d_Hk%d_d%d_T%d_L%d" % c)
def test_bwd_bf16_small(case):
    w = small_w(*case, backward=True)
    x = I.make_inputs(w, device=DEV)
    out = run_gpu(w, x)
    ref = oracle_bwd_full(w, x)
    for name, r in zip(("dQ", "dK", "dV", "dKd", "dVd"), ref):
        if out[name] is None:
            assert r.size == 0
            continue
        assert_grad_close(f64(out[name]), r, name)


def test_bwd_fp32_tiny():
    w = I.TINY_FP32.with_(backward=True)
    x = I.make_inputs(w, device=DEV)
    out = run_gpu(w, x)
    ref = oracle_bwd_full(w, x)
    for name, r in zip(("dQ", "dK", "dV", "dKd", "dVd"), ref):
        assert err_stats(f64(out[name]), r)[0] <= 1e-4, name


def _check_slices(w, x, out, slices):
    for (b, hk) in slices:
        ws, xs = slice_workload(w, x, b, hk)
        ref = oracle_bwd_full(ws, xs)
        G = w.G
        got = {"dQ": out["dQ"][b:b + 1, hk * G:(hk + 1) * G], "dK": out["dK"][b:b + 1, hk:hk + 1],
               "dV": out["dV"][b:b + 1, hk:hk + 1], "dKd": out["dKd"][b:b + 1, hk:hk + 1],
               "dVd": out["dVd"][b:b + 1, hk:hk + 1]}
        for name, r in zip(("dQ", "dK", "dV", "dKd", "dVd"), ref):
            assert_grad_close(f64(got[name]), r, f"{w.name} slice ({b},{hk}) {name}")


def test_bwd_layer_T4k_sampled_slices():
    w = I.LAYER_1P5B
    x = I.make_inputs(w, device=DEV)
    out = run_gpu(w, x)
    _check_rows(w, x, out)
    _check_slices(w, x, out, [(0, 0), (0, 2), (1, 1), (w.B - 1, w.Hk - 1)])


def test_bwd_train_shape_sampled_slice():
    w = I.TRAIN_FWD_BWD
    x = I.make_inputs(w, device=DEV)
    out = run_gpu(w, x)
    _check_slices(w, x, out, [(0, 0), (2, 6), (5, 3), (w.B - 1, w.Hk - 1)])


def test_bwd_deterministic():
    w = small_w(1, 8, 2, 128, 300, 6, backward=True)
    x = I.make_inputs(w, device=DEV)
    a = run_gpu(w, x)
    b = run_gpu(w, x)
    for k in ("dQ", "dK", "dV", "dKd", "dVd"):
        assert torch.equal(a[k], b[k]), k


# (B, Hq, Hk, d, T, L, causal, window): every G the stored-dS backward takes
# (1, 2, 4, 8), ragged T, the modes; G = 3 and d = 64 fall back to recomputing
BOTH_PATHS = [
    (1, 4, 4, 128, 300, 5, True, 0),      # G = 1: 128 tokens per query tile
    (2, 4, 2, 128, 257, 3, True, 0),      # G = 2
    (1, 8, 2, 128, 513, 16, True, 0),     # G = 4
    (1, 16, 2, 128, 200, 6, True, 0),     # G = 8: 16 tokens per query tile
    (1, 8, 2, 128, 300, 8, False, 3),     # non-causal, depth window
    (1, 8, 1, 128, 129, 0, True, 0),      # L = 0, ragged last tile of 128 tokens
    (1, 6, 2, 128, 100, 5, True, 0),      # G = 3: no stored path
    (1, 8, 2, 64, 200, 4, True, 0),       # d = 64: no stored path
]


@pytest.mark.parametrize("case", BOTH_PATHS, ids=lambda c: "B%d_Hq%d_Hk%d_d%d_T%d_L%d_c%d_w%d" % c)
def test_bwd_stored_and_recomputed_paths(case):
    """The backward with its full workspace (dS stored by the dK/dV kernel,
    read by the dQ kernel) and with the least workspace (dQ kernel
    recomputes S and dP): both match the oracle, the workspace guards hold,
    and each is bitwise repeatable."""
    B, Hq, Hk, d, T, L, causal, window = case
    w = small_w(B, Hq, Hk, d, T, L, backward=True).with_(causal=causal, window=window)
    x = I.make_inputs(w, device=DEV)
    ref = oracle_bwd_full(w, x)
    for mode in (1, 2):
        out = run_gpu(w, x, ws_mode=mode)
        for name, r in zip(("dQ", "dK", "dV", "dKd", "dVd"), ref):
            if out[name] is None:
                assert r.size == 0
                continue
            assert_grad_close(f64(out[name]), r, f"ws_mode {mode} {name}")
        again = run_gpu(w, x, ws_mode=mode)
        for name in ("dQ", "dK", "dV", "dKd", "dVd"):
            if out[name] is not None:
                assert torch.equal(out[name], again[name]), f"ws_mode {mode} {name} not repeatable"


def test_bwd_workspace_error_on_device():
    w = small_w(1, 4, 2, 128, 64, 2, backward=True)
    x = I.make_inputs(w, device=DEV)
    out = run_gpu(w, x, backward=False)
    sh = moda.make_shape(w.B, w.Hq, w.Hk, w.T, w.d, w.L, w.C)
    need = moda.moda_workspace_size(sh, 2)
    ws = torch.empty(need, device=DEV, dtype=torch.uint8)
    g = {k: torch.empty_like(v) for k, v in (("dQ", x["Q"]), ("dK", x["K"]), ("dV", x["V"]),
                                            ("dKd", out["Kd"]), ("dVd", out["Vd"]))}
    with pytest.raises(moda.MoDAError) as ei:
        moda.moda_bwd(sh, x["Q"], x["K"], x["V"], out["Kd"], out["Vd"], out["O"], out["LSE"],
                      x["dO"], g["dQ"], g["dK"], g["dV"], g["dKd"], g["dVd"], ws, need - 16)
    assert ei.value.status == 4


# ------------------------------------------- non-causal and depth window ----
MODES = [(False, 0), (True, 3), (False, 2), (True, 8)]
MODE_CASES = [(1, 8, 2, 128, 300, 8), (2, 4, 4, 64, 130, 5), (1, 6, 2, 128, 97, 3)]


@pytest.mark.parametrize("mode", MODES, ids=lambda m: "causal%d_win%d" % m)
@pytest.mark.parametrize("case", MODE_CASES, ids=lambda c: "B%d_Hq%d_Hk%d_d%d_T%d_L%d" % c)
def test_modes_fwd_bwd_small(case, mode):
    causal, window = mode
    if window > case[5]:
        pytest.skip("window larger than L")
    w = small_w(*case, backward=True).with_(causal=causal, window=window)
    x = I.make_inputs(w, device=DEV)
    out = run_gpu(w, x)
    O, LSE = oracle_fwd_full(w, x)
    assert_out_close(f64(out["O"]), O, "bf16", "O")
    assert err_stats(f64(out["LSE"]), LSE)[0] <= LSE_MAX_ABS
    for name, r in zip(("dQ", "dK", "dV", "dKd", "dVd"), oracle_bwd_full(w, x)):
        assert_grad_close(f64(out[name]), r, name)


def test_modes_fp32():
    for causal, window in MODES:
        w = I.TINY_FP32.with_(causal=causal, window=window, backward=True)
        x = I.make_inputs(w, device=DEV)
        out = run_gpu(w, x)
        O, _ = oracle_fwd_full(w, x)
        assert_out_close(f64(out["O"]), O, "fp32", f"O causal={causal} window={window}")
        for name, r in zip(("dQ", "dK", "dV", "dKd", "dVd"), oracle_bwd_full(w, x)):
            assert err_stats(f64(out[name]), r)[0] <= 1e-4, name


def test_modes_layer_T4k_sampled():
    for causal, window in ((False, 0), (True, 4)):
        w = I.LAYER_1P5B.with_(causal=causal, window=window)
        x = I.make_inputs(w, device=DEV)
        out = run_gpu(w, x)
        _check_rows(w, x, out)
        _check_slices(w, x, out, [(0, 2)])


def test_fwd_bwd_many_tiles_per_cta():
    """512 short query tiles: the forward runs persistent CTAs that each walk
    several tiles (ring phases and the Q / O hand-offs cross tile boundaries);
    checked in full, with a ragged last tile (T = 1000)."""
    w = small_w(4, 16, 8, 64, 1000, 6, backward=True)
    x = I.make_inputs(w, device=DEV)
    out = run_gpu(w, x)
    O, LSE = oracle_fwd_full(w, x)
    assert_out_close(f64(out["O"]), O, "bf16", "O")
    assert err_stats(f64(out["LSE"]), LSE)[0] <= LSE_MAX_ABS
    for name, r in zip(("dQ", "dK", "dV", "dKd", "dVd"), oracle_bwd_full(w, x)):
        assert_grad_close(f64(out[name]), r, name)


# (B, Hq, Hk, d, T, L): stored dS with more tiles than SMs and ragged ends.
# The first case has 216 key tiles, so the dK/dV kernel runs persistent CTAs
# that walk several key tiles each (ring, TMEM-buffer and accumulator phases
# cross item boundaries); all three have more query tiles than SMs, with a
# ragged last query tile whose stored dS rows past T are never written.
PERSISTENT_BWD = [
    (3, 16, 8, 128, 1100, 5),     # G = 2: 216 key tiles, 432 query tiles
    (2, 16, 4, 128, 1200, 7),     # G = 4: 304 query tiles, the last one half full
    (1, 16, 2, 128, 1300, 3),     # G = 8: 164 query tiles of 16 tokens
]


@pytest.mark.parametrize("case", PERSISTENT_BWD, ids=lambda c: "B%d_Hq%d_Hk%d_d%d_T%d_L%d" % c)
def test_bwd_persistent_tiles(case):
    w = small_w(*case, backward=True)
    x = I.make_inputs(w, device=DEV)
    out = run_gpu(w, x, ws_mode=1)
    for name, r in zip(("dQ", "dK", "dV", "dKd", "dVd"), oracle_bwd_full(w, x)):
        assert_grad_close(f64(out[name]), r, name)
    again = run_gpu(w, x, ws_mode=1)
    for name in ("dQ", "dK", "dV", "dKd", "dVd"):
        assert torch.equal(out[name], again[name]), f"{name} not repeatable"


# (B, Hq, Hk, d, T, L, causal, window): the layer-major depth layout, read in
# place through 4-D tensor-map views (no repack), against the flat layout
LAYER_CASES = [
    (1, 8, 2, 128, 513, 16, True, 0),     # G = 4, ragged last tile
    (2, 4, 4, 128, 300, 8, True, 0),      # G = 1: 128 tokens per query tile
    (1, 16, 2, 128, 200, 3, True, 0),     # G = 8: 48-row depth blocks of 16 tokens
    (2, 4, 2, 64, 257, 4, True, 0),       # d = 64: the recomputing dQ kernel
    (1, 8, 2, 128, 300, 8, False, 3),     # non-causal, depth window
    (1, 6, 2, 128, 100, 2, True, 0),      # G = 3: head-major rows, recomputing dQ
]


@pytest.mark.parametrize("case", LAYER_CASES, ids=lambda c: "B%d_Hq%d_Hk%d_d%d_T%d_L%d_c%d_w%d" % c)
def test_layer_layout_small(case):
    """The layer-major cache read in place gives the flat layout's results bit
    for bit (the same shared-memory depth tiles), dK_d / dV_d written back
    layer-major; both backward workspaces; and the oracle agrees."""
    B, Hq, Hk, d, T, L, causal, window = case
    w = small_w(B, Hq, Hk, d, T, L, backward=True).with_(causal=causal, window=window)
    x = I.make_inputs(w, device=DEV)
    for mode in (1, 2):
        flat = run_gpu(w, x, ws_mode=mode)
        lay = run_gpu(w, x, layout=moda.MODA_DEPTH_LAYER, ws_mode=mode)
        for k in ("O", "LSE", "dQ", "dK", "dV", "dKd", "dVd"):
            assert torch.equal(flat[k], lay[k]), f"ws_mode {mode} {k}"
    O, LSE = oracle_fwd_full(w, x)
    assert_out_close(f64(lay["O"]), O, "bf16", "O")
    for name, r in zip(("dQ", "dK", "dV", "dKd", "dVd"), oracle_bwd_full(w, x)):
        assert_grad_close(f64(lay[name]), r, name)


def test_layer_layout_full_size():
    """layer_1p5b_T4k with the layer-major cache: bitwise the flat layout's
    outputs and gradients (the launch configuration the benchmark times)."""
    w = I.LAYER_1P5B
    x = I.make_inputs(w, device=DEV)
    flat = run_gpu(w, x)
    lay = run_gpu(w, x, layout=moda.MODA_DEPTH_LAYER)
    for k in ("O", "LSE", "dQ", "dK", "dV", "dKd", "dVd"):
        assert torch.equal(flat[k], lay[k]), k


def test_layer_layout_long_context_forward():
    """long_context_T64k forward from the layer-major cache (1 KB per layer
    plane per depth block): bitwise the flat layout's O and LSE."""
    w = I.LONG_64K
    x = I.make_inputs(w, device=DEV, grad_out=False)
    flat = run_gpu(w, x, backward=False)
    lay = run_gpu(w, x, backward=False, layout=moda.MODA_DEPTH_LAYER)
    assert torch.equal(flat["O"], lay["O"]) and torch.equal(flat["LSE"], lay["LSE"])


def test_bench_step_every_slice():
    """layer_1p5b_T4k exactly as the benchmark step runs it (layer-major depth
    caches read in place, full backward workspace): O, LSE and all five
    gradients of every (b, hk) slice against the oracle."""
    w = I.LAYER_1P5B
    x = I.make_inputs(w, device=DEV)
    out = run_gpu(w, x, layout=moda.MODA_DEPTH_LAYER, ws_mode=1)
    G = w.G
    for b in range(w.B):
        for hk in range(w.Hk):
            ws, xs = slice_workload(w, x, b, hk)
            O, LSE = oracle_fwd_full(ws, xs)
            assert_out_close(f64(out["O"][b:b + 1, hk * G:(hk + 1) * G]), O, "bf16", f"slice ({b},{hk}) O")
            assert err_stats(f64(out["LSE"][b:b + 1, hk * G:(hk + 1) * G]), LSE)[0] <= LSE_MAX_ABS
            got = {"dQ": out["dQ"][b:b + 1, hk * G:(hk + 1) * G], "dK": out["dK"][b:b + 1, hk:hk + 1],
                   "dV": out["dV"][b:b + 1, hk:hk + 1], "dKd": out["dKd"][b:b + 1, hk:hk + 1],
                   "dVd": out["dVd"][b:b + 1, hk:hk + 1]}
            for name, r in zip(("dQ", "dK", "dV", "dKd", "dVd"), oracle_bwd_full(ws, xs)):
                assert_grad_close(f64(got[name]), r, f"slice ({b},{hk}) {name}")


def test_layer_layout_persistent_and_modes():
    """Layer-major caches with persistent dK/dV (216 key tiles), more query
    tiles than SMs and a ragged end, causal and non-causal with a depth
    window: bitwise the flat layout, and the oracle agrees."""
    for causal, window in ((True, 0), (False, 3)):
        w = small_w(3, 16, 8, 128, 1100, 4, backward=True).with_(causal=causal, window=window)
        x = I.make_inputs(w, device=DEV)
        flat = run_gpu(w, x, ws_mode=1)
        lay = run_gpu(w, x, layout=moda.MODA_DEPTH_LAYER, ws_mode=1)
        for k in ("O", "LSE", "dQ", "dK", "dV", "dKd", "dVd"):
            assert torch.equal(flat[k], lay[k]), f"causal={causal} {k}"
        O, _ = oracle_fwd_full(w, x)
        assert_out_close(f64(lay["O"]), O, "bf16", f"causal={causal} O")
        for name, r in zip(("dQ", "dK", "dV", "dKd", "dVd"), oracle_bwd_full(w, x)):
            assert_grad_close(f64(lay[name]), r, f"causal={causal} {name}")
