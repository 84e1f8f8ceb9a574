"""The oracle against its pins (CPU only)."""
import pytest

import oracle
from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oracle)


def test_keep_count_rejects_bad_sparsity():
    for s in (-0.1, 1.0, 1.5):
        with pytest.raises(ValueError):
            oracle.keep_count(128, s)
