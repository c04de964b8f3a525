"""The oracle against facts fixed outside it (see tests/oracle_pins.py for each source)."""
import pytest

import oracle
import oracle_pins


@pytest.fixture(scope="module")
def lib():
    return oracle.load_library()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, lib):
    pin(lib)


def test_backward_finite_differences_T128(lib):
    """The training-step workload's check: finite differences at T=128 (two chunks of 64)."""
    oracle_pins.pin_backward_finite_differences(lib, T=128, dk=16, dv=16, ndir=2)
