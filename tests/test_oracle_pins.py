"""The float64 oracle against its pins (closed forms, hand-worked cases,
brute force, invariants).  CPU only."""
import pytest

from oracle import oracle
import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.lib())


@pytest.mark.parametrize("pin", oracle_pins.QPINS, ids=lambda f: f.__name__)
def test_quantizer_pin(pin):
    pin(oracle.quantize_keys)
