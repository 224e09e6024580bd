"""The worked example in tests/golden: a MoDA forward and backward whose
values are exact fractions (or fractions of ln 2) taken straight from the
operator's definition by tests/golden/make_worked_example.py, which shares no
code with the oracle or the library.  It fixes, by value, the 1/sqrt(d)
scale, the causal boundary j <= t, that a token sees only its own depth rows,
the joint normalisation over both, the floor(h/G) head map and the routing of
every gradient (depth gradients token-local).  Checked against the oracle on
the CPU (fp64) and against the CUDA fp32 path on the GPU."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from worked_example import GOLD, load


def test_fixture_matches_generator():
    """The committed fixture is what the exact generator writes."""
    import subprocess
    import sys
    import tempfile
    gen = os.path.join(os.path.dirname(GOLD), "make_worked_example.py")
    with tempfile.TemporaryDirectory() as tmp:
        src = open(gen).read()
        path = os.path.join(tmp, "make_worked_example.py")
        open(path, "w").write(src)
        subprocess.run([sys.executable, path], check=True, capture_output=True)
        fresh = json.load(open(os.path.join(tmp, "worked_example_G2_T3_L2.json")))
    assert fresh == json.load(open(GOLD))


def test_oracle_reproduces_worked_example():
    x, e = load()
    lib = oracle.load_library()
    O, LSE = oracle.fwd(x["Q"], x["K"], x["V"], x["Kd"], x["Vd"], lib=lib)
    np.testing.assert_allclose(O, e["O"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSE, e["LSE"], rtol=0, atol=1e-12)
    grads = oracle.bwd(x["Q"], x["K"], x["V"], x["Kd"], x["Vd"], x["dO"], lib=lib)
    for name, got in zip(("dQ", "dK", "dV", "dKd", "dVd"), grads):
        np.testing.assert_allclose(got, e[name], rtol=0, atol=1e-12, err_msg=name)


@pytest.mark.gpu
def test_cuda_fp32_path_reproduces_worked_example():
    import sequence_depth_attention_moda_b200 as moda
    from moda_cases import FP32_MAX_ABS, Guarded
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    x, e = load()
    s = x["shape"]
    B, Hq, Hk, T, L, d = s["B"], s["Hq"], s["Hk"], s["T"], s["L"], s["d"]
    dev = lambda a: torch.tensor(a, dtype=torch.float32, device="cuda").contiguous()
    Q, K, V, dO = dev(x["Q"]), dev(x["K"]), dev(x["V"]), dev(x["dO"])
    Kd, Vd = dev(x["Kd"]), dev(x["Vd"])
    sh = moda.make_shape(B, Hq, Hk, T, d, L, 0, moda.MODA_FP32)
    gd = Guarded()
    O = gd.like("O", Q)
    LSE = gd.empty("LSE", (B, Hq, T), torch.float32, "cuda")
    moda.moda_fwd(sh, Q, K, V, Kd, Vd, O, LSE)
    nws = moda.moda_workspace_size(sh, True)
    ws = torch.empty(max(nws, 16), device="cuda", dtype=torch.uint8)
    g = [gd.like(n, t) for n, t in zip(("dQ", "dK", "dV", "dKd", "dVd"), (Q, K, V, Kd, Vd))]
    moda.moda_bwd(sh, Q, K, V, Kd, Vd, O, LSE, dO, *g, ws, nws)
    moda.moda_check_status()
    gd.check()
    got = {"O": O, "LSE": LSE, "dQ": g[0], "dK": g[1], "dV": g[2], "dKd": g[3], "dVd": g[4]}
    for name, t in got.items():
        np.testing.assert_allclose(t.double().cpu().numpy(), e[name], rtol=0, atol=FP32_MAX_ABS,
                                   err_msg=name)
