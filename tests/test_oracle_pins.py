"""The CPU oracle against its pins (closed forms, hand values, brute force).

Parity status: every oracle entry point (prefill rows in landmark, given and
exact-mass modes; decode; decode over a paged cache; union) is pinned here;
none is unpinned.  The pages
print no worked numeric example, so the pins are closed forms and hand-derived
values listed in tests/pins.py with the passage each one follows.
"""
import pytest

import oracle
from tests import pins


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)
