"""The fp64 oracle against closed forms, brute force, the pages' chunkwise
algorithm and invariants (CPU only)."""
import pytest

import oracle
import pins


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@pytest.mark.parametrize("name,pin", pins.all_pins(), ids=[n for n, _ in pins.all_pins()])
def test_pin(lib, name, pin):
    err = pin(lib)
    assert err <= pins.PIN_TOL, f"{name}: error {err:.3e}"
