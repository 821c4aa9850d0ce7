"""The fp64 oracle against closed forms, invariants, finite differences, hand-worked examples and a
float64 library routine (CPU only)."""
import pytest

import oracle_pins


@pytest.fixture(scope="module")
def orc():
    import oracle

    return oracle.Oracle()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_rejects_bad_rows(orc):
    import numpy as np

    q = np.zeros((1, 4, 2))
    with pytest.raises(ValueError):
        orc.fwd(q, q, q, rows=np.array([[4]]))
    with pytest.raises(ValueError):
        orc.fwd(q, q, q, rows=np.array([[-1]]))
