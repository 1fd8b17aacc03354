"""The fp64 oracle against facts fixed by the pages and by mathematics."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import oracle_pins  # noqa: E402
from oracle import mla_oracle  # noqa: E402


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(mla_oracle)
