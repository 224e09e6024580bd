"""moda_bwd_noalloc: the backward for callers that cannot allocate device
memory where they run it (a plugin whose host framework forbids allocation
during execution, code replaying a fixed memory plan).  Its scratch is a fixed
array inside the library instead of a caller workspace.

The results must match moda_bwd (the entry point that takes a workspace) on
two calls in a row with different inputs, so scratch contents left behind by
the first call cannot leak into the second.  This file is collected last.
"""
import pytest
import torch

import sequence_depth_attention_moda_b200 as moda
from sequence_depth_attention_moda_b200 import inputs as I
from moda_cases import assert_grad_close, f64, run_gpu, shape_of

pytestmark = pytest.mark.gpu

W = I.Workload("noalloc", B=2, Hq=8, Hk=2, d=128, T=700, L=6, C=1, backward=True, seed=4242)


def _grads_noalloc(w, x, fwd):
    sh = shape_of(w)
    g = {"dQ": torch.empty_like(x["Q"]), "dK": torch.empty_like(x["K"]),
         "dV": torch.empty_like(x["V"]), "dKd": torch.empty_like(fwd["Kd"]),
         "dVd": torch.empty_like(fwd["Vd"])}
    moda.moda_bwd_noalloc(sh, x["Q"], x["K"], x["V"], fwd["Kd"], fwd["Vd"], fwd["O"], fwd["LSE"],
                          x["dO"], g["dQ"], g["dK"], g["dV"], g["dKd"], g["dVd"])
    return g


def test_noalloc_matches_workspace_backward_twice():
    assert torch.cuda.is_available(), "CUDA device required"
    for call, seed in enumerate((4242, 4343)):
        w = W.with_(seed=seed)
        x = I.make_inputs(w, device="cuda")
        ref = run_gpu(w, x)                      # repack + forward + moda_bwd with a workspace
        got = _grads_noalloc(w, x, ref)
        torch.cuda.synchronize()
        moda.moda_check_status()
        for k in ("dQ", "dK", "dV", "dKd", "dVd"):
            assert_grad_close(f64(got[k]), f64(ref[k]), f"call {call} {k}")


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 4,194,305 query rows > the 4,194,304-row built-in scratch: rejected
    # before anything is queued (the pointers are never touched).
    sh = moda.make_shape(1, 1, 1, 4194305, 128, 0, 0)
    fake = 1 << 20
    with pytest.raises(moda.MoDAError) as ei:
        moda.moda_bwd_noalloc(sh, fake, fake, fake, None, None, fake, fake, fake, fake, fake,
                              fake, None, None, stream=0)
    assert ei.value.status == 4 and "scratch" in str(ei.value)
