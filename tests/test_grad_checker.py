"""The gradient checker itself, on the CPU: its bounds must reject plausible
wrong gradients at the magnitudes of the 1.5B-scale layer workload (Q, K and
K_depth drawn as N(0,1)/sqrt(d), so the gradients are small and spread over
orders of magnitude), and must accept what bf16 storage of the exact
gradients gives.  The reference gradients are the oracle's, on one (b, hk)
slice of that workload shortened to T = 512."""
import numpy as np
import pytest
import torch

from moda_cases import assert_grad_close, f64, oracle_bwd_full, slice_workload
from sequence_depth_attention_moda_b200 import inputs as I

NAMES = ("dQ", "dK", "dV", "dKd", "dVd")


@pytest.fixture(scope="module")
def grads():
    w = I.LAYER_1P5B.with_(T=512)
    x = I.make_inputs(w, device="cpu")
    ws, xs = slice_workload(w, x, 0, 0)
    return ws, dict(zip(NAMES, oracle_bwd_full(ws, xs)))


def _bf16(a):
    return f64(torch.from_numpy(a).to(torch.bfloat16))


def _fails(got, ref, name):
    with pytest.raises(AssertionError):
        assert_grad_close(got, ref, name)


def test_exact_and_bf16_rounded_gradients_pass(grads):
    _, g = grads
    for name in NAMES:
        assert_grad_close(g[name], g[name], name)
        assert_grad_close(_bf16(g[name]), g[name], name + " (bf16)")


@pytest.mark.parametrize("name", NAMES)
def test_five_percent_scale_error_fails(grads, name):
    _, g = grads
    _fails(1.05 * g[name], g[name], name)


@pytest.mark.parametrize("name", NAMES)
def test_all_zero_gradient_fails(grads, name):
    _, g = grads
    _fails(np.zeros_like(g[name]), g[name], name)


def test_one_token_of_depth_gradients_zeroed_fails(grads):
    ws, g = grads
    for name in ("dKd", "dVd"):
        bad = g[name].copy()
        bad[:, :, 0:ws.L] = 0.0                  # token 0's L depth rows
        _fails(bad, g[name], name)


def test_depth_gradients_of_the_neighbouring_token_fail(grads):
    ws, g = grads
    for name in ("dKd", "dVd"):
        bad = np.roll(g[name], ws.L, axis=2)     # token t's rows hold token t-1's
        _fails(bad, g[name], name)


def test_sign_flip_of_one_head_fails(grads):
    _, g = grads
    bad = g["dQ"].copy()
    bad[:, 1] *= -1.0
    _fails(bad, g["dQ"], "dQ")


def test_zero_reference_demands_exact_zeros():
    ref = np.zeros((2, 3))
    assert_grad_close(ref.copy(), ref, "zeros")
    _fails(np.full((2, 3), 1e-30), ref, "zeros")
