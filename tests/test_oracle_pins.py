"""The fp64 oracle against its pins (brute force, exact rationals, closed forms,
invariants). CPU only."""
import pytest

from tests import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(oracle, pin):
    pin(oracle)


def test_tiny_has_zero_rows(oracle):
    """The tiny workload's eight forced rows really have phi(Q) = 0 in every
    head (so its eps path is exercised), and no other row does."""
    import numpy as np
    (Q, K, V), eps = pins.tiny_inputs()
    _, den = oracle.forward(Q, K, V, eps, return_den=True)
    zero_rows = sorted(set(np.nonzero(den[0] == 0)[0].tolist()))
    assert zero_rows == [0, 37, 74, 111, 148, 185, 222, 255]
