"""The CPU oracle against closed forms, invariants, library routines and hand-worked examples."""

import pytest

import oracle_pins as P


@pytest.mark.parametrize("pin", P.ATTENTION_PINS + P.PLAN_PINS, ids=lambda f: f.__name__)
def test_pin(pin, oracle_lib):
    pin()
