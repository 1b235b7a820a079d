"""The fp64 oracle against its pins (CPU only). See ``oracle_pins.py``."""

import pytest

import oracle_pins


@pytest.mark.parametrize("name", list(oracle_pins.PINS))
def test_pin(name):
    ok, detail = oracle_pins.PINS[name]()
    assert ok, f"{name}: {detail}"
