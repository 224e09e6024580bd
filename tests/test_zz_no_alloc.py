"""moda_bwd_noalloc: the backward for callers that cannot allocate device
memory where they run it (a plugin whose host framework forbids allocation
during execution, code replaying a fixed memory plan).  Its scratch is a fixed
array inside the library instead of a caller workspace.

It runs the same kernels as moda_bwd given the least workspace moda_bwd
accepts (moda_workspace_size(shape, 2): the dQ kernel recomputes S and dP), so
its results must be bit-identical to those, on two calls in a row with
different inputs (scratch contents left behind by the first call must not leak
into the second), for the tensor-core bf16 path and the CUDA-core fp32 path;
and within the gradient tolerance of moda_bwd with its full workspace (the
stored-dS path).  This file is collected last.
"""
import pytest
import torch

import sequence_depth_attention_moda_b200 as moda
from sequence_depth_attention_moda_b200 import inputs as I
from moda_cases import Guarded, assert_grad_close, f64, run_gpu, shape_of

pytestmark = pytest.mark.gpu

NAMES = ("dQ", "dK", "dV", "dKd", "dVd")
W_BF16 = I.Workload("noalloc", B=2, Hq=8, Hk=2, d=128, T=700, L=6, C=1, backward=True, seed=4242)
W_FP32 = I.TINY_FP32.with_(backward=True, seed=4244)


def _grads_noalloc(w, x, fwd):
    sh = shape_of(w)
    gd = Guarded()
    g = {"dQ": gd.like("dQ", x["Q"]), "dK": gd.like("dK", x["K"]), "dV": gd.like("dV", x["V"]),
         "dKd": gd.like("dKd", fwd["Kd"]), "dVd": gd.like("dVd", fwd["Vd"])}
    moda.moda_bwd_noalloc(sh, x["Q"], x["K"], x["V"], fwd["Kd"], fwd["Vd"], fwd["O"], fwd["LSE"],
                          x["dO"], g["dQ"], g["dK"], g["dV"], g["dKd"], g["dVd"])
    gd.check()
    return g


@pytest.mark.parametrize("w", [W_BF16, W_FP32], ids=["bf16", "fp32"])
def test_noalloc_matches_workspace_backward_twice(w):
    assert torch.cuda.is_available(), "CUDA device required"
    for call, seed in enumerate((w.seed, w.seed + 101)):
        wc = w.with_(seed=seed)
        x = I.make_inputs(wc, device="cuda")
        ref = run_gpu(wc, x, ws_mode=2)          # repack + forward + moda_bwd, least workspace
        fast = run_gpu(wc, x, ws_mode=1)         # moda_bwd with its full workspace
        got = _grads_noalloc(wc, x, ref)
        torch.cuda.synchronize()
        moda.moda_check_status()
        for k in NAMES:
            assert torch.equal(got[k], ref[k]), f"call {call} {k}: differs from moda_bwd"
            assert_grad_close(f64(got[k]), f64(fast[k]), f"call {call} {k} vs the stored-dS path")


def test_noalloc_layer_major_depth():
    """With the layer-major depth layout (caches read in place, dKd / dVd
    written layer-major) the no-allocation backward gives moda_bwd's bits."""
    w = W_BF16.with_(L=8)
    x = I.make_inputs(w, device="cuda")
    ref = run_gpu(w, x, layout=moda.MODA_DEPTH_LAYER, ws_mode=2)
    sh = shape_of(w, moda.MODA_DEPTH_LAYER)
    gd = Guarded()
    g = {"dQ": gd.like("dQ", x["Q"]), "dK": gd.like("dK", x["K"]), "dV": gd.like("dV", x["V"]),
         "dKd": gd.like("dKd", x["Kd_layer"]), "dVd": gd.like("dVd", x["Vd_layer"])}
    moda.moda_bwd_noalloc(sh, x["Q"], x["K"], x["V"], x["Kd_layer"], x["Vd_layer"], ref["O"], ref["LSE"],
                          x["dO"], g["dQ"], g["dK"], g["dV"], g["dKd"], g["dVd"])
    gd.check()
    torch.cuda.synchronize()
    moda.moda_check_status()
    for k in ("dQ", "dK", "dV"):
        assert torch.equal(g[k], ref[k]), k
    assert torch.equal(g["dKd"], ref["dKd_layer"]) and torch.equal(g["dVd"], ref["dVd_layer"])


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 4,194,305 query rows > the 4,194,304-row built-in scratch: rejected
    # before anything is queued (the pointers are never touched).
    sh = moda.make_shape(1, 1, 1, 4194305, 128, 0, 0)
    fake = 1 << 20
    with pytest.raises(moda.MoDAError) as ei:
        moda.moda_bwd_noalloc(sh, fake, fake, fake, None, None, fake, fake, fake, fake, fake,
                              fake, None, None, stream=0)
    assert ei.value.status == moda.MODA_ERR_WORKSPACE and "scratch" in str(ei.value)


def test_noalloc_pointer_errors_match_moda_bwd():
    # Rejected on the host before anything is queued: a misaligned depth
    # pointer is MODA_ERR_MISALIGNED, a NULL one MODA_ERR_INVALID_ARG, as for
    # moda_bwd.  The (aligned) fake addresses are never dereferenced.
    sh = moda.make_shape(1, 2, 1, 64, 128, 4, 0)
    fake = 1 << 20
    for bad, status in ((fake + 8, moda.MODA_ERR_MISALIGNED), (None, moda.MODA_ERR_INVALID_ARG)):
        for entry in ("noalloc", "bwd"):
            with pytest.raises(moda.MoDAError) as ei:
                if entry == "noalloc":
                    moda.moda_bwd_noalloc(sh, fake, fake, fake, bad, fake, fake, fake, fake, fake,
                                          fake, fake, fake, fake, stream=0)
                else:
                    moda.moda_bwd(sh, fake, fake, fake, bad, fake, fake, fake, fake, fake, fake,
                                  fake, fake, fake, fake, 1 << 30, stream=0)
            assert ei.value.status == status, (entry, bad)
