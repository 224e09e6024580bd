"""The CPU oracle against its pins (no GPU).  See ``oracle_pins.py``."""
import numpy as np
import pytest

import oracle
import oracle_pins


@pytest.fixture(scope="module")
def lib():
    return oracle.load_library()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(lib, pin):
    pin(lib)


def test_row_entry_point_matches_full_forward(lib):
    """The single-row entry point (used for sampled rows at full size) gives
    the same numbers as the full forward."""
    Q, K, V, Kd, Vd, _ = oracle_pins.rand_case(1, 4, 2, 9, 8, 3, 5)
    O, LSE = oracle.fwd(Q, K, V, Kd, Vd, lib=lib)
    for (h, t) in ((0, 0), (3, 8), (1, 4)):
        hk = h // 2
        o, lse = oracle.row(Q[0, h, t], K[0, hk, :t + 1], V[0, hk, :t + 1],
                            Kd[0, hk, t * 3:(t + 1) * 3], Vd[0, hk, t * 3:(t + 1) * 3], lib=lib)
        assert np.array_equal(o, O[0, h, t]) and lse == LSE[0, h, t]


def test_rejects_bad_shape(lib):
    Q, K, V, Kd, Vd, _ = oracle_pins.rand_case(1, 3, 2, 4, 8, 1, 6)
    with pytest.raises(ValueError):
        oracle.fwd(Q, K, V, Kd, Vd, lib=lib)   # Hq % Hk != 0
