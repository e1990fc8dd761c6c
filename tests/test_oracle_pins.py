"""The fp64 oracle against what the pages and the mathematics fix (CPU only)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    err, tol = pin()
    assert err <= tol, f"{pin.__name__}: error {err:.3e} > {tol:.1e}"


def test_golden_file_has_cases():
    names = [c["name"] for c in oracle_pins.load_golden()]
    assert len(names) >= 4 and len(set(names)) == len(names)
