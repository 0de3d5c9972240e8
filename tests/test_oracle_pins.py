"""The CPU oracle against closed forms, hand-derived values, torch fp64 and
finite differences (no GPU)."""

import pytest

import oracle
import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.default())


def test_oracle_rejects_bad_shapes():
    import numpy as np
    q = np.zeros((1, 3, 4, 2))
    k = np.zeros((1, 2, 4, 2))
    with pytest.raises(ValueError):
        oracle.fwd(q, k, k, 1.0, False)
    with pytest.raises(ValueError):
        oracle.fwd_rows(q[:, :2], k, k, [4], 1.0, False)


def test_oracle_empty_sequence():
    import numpy as np
    q = np.zeros((1, 2, 0, 8))
    o, lse = oracle.fwd(q, q, q, 1.0, True)
    assert o.shape == (1, 2, 0, 8) and lse.shape == (1, 2, 0)
