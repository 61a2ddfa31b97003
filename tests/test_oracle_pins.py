"""The FP64 oracle against its pins (closed forms, invariants, brute force,
library routines); see oracle_pins.py for what each pin fixes."""
import pytest

import oracle
import oracle_pins as P


class _Real:
    attn_fwd = staticmethod(oracle.attn_fwd)
    rope = staticmethod(oracle.rope)


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(_Real)
