"""The kernels' bounded-wait failure path, made to run without any fault.

moda_selftest_wait_timeout queues one CTA whose warps wait, through the same
bounded mbarrier wait as the forward and backward kernels, on a barrier that
nothing arrives on.  The wait must give up, the status word must carry the
timeout to the host exactly once, and the device must stay usable.
"""
import time

import pytest
import torch

import sequence_depth_attention_moda_b200 as moda
from sequence_depth_attention_moda_b200 import inputs as I
from moda_cases import assert_out_close, f64, oracle_fwd_full, run_gpu

pytestmark = pytest.mark.gpu


def test_wait_timeout_reported_and_device_usable():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    moda.moda_check_status()                      # start from a clear word
    t0 = time.monotonic()
    moda.moda_selftest_wait_timeout()
    with pytest.raises(moda.MoDAError) as err:
        moda.moda_check_status()
    elapsed = time.monotonic() - t0
    assert err.value.status == moda.MODA_ERR_TIMEOUT
    assert 1.5 < elapsed < 30.0, elapsed          # the 2 s limit, not a hang
    moda.moda_check_status()                      # the word was cleared
    # the context still runs the operator correctly
    w = I.TINY_FP32
    x = I.make_inputs(w, device="cuda")
    out = run_gpu(w, x)
    O, _ = oracle_fwd_full(w, x)
    assert_out_close(f64(out["O"]), O, "fp32", "O after a timeout")
    moda.moda_check_status()
