"""The fp64 oracle against what the pages and mathematics fix (CPU only)."""
import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.fixture(scope="module")
def lib():
    return oracle._get_lib()


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, lib):
    pin(lib)


def test_rel_err_metric():
    import numpy as np
    ref = np.array([1.0, -1.0, 1.0, -1.0])
    assert oracle.rel_err(ref + np.array([0, 0, 0.5, 0]), ref) == pytest.approx(0.5)
    assert oracle.rel_err(np.zeros(0), np.zeros(0)) == 0.0
