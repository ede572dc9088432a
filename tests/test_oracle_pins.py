"""The CPU oracle against facts that do not come from itself (CPU only)."""
import pytest

import oracle
from tests import oracle_pins


@pytest.fixture(scope="module")
def o():
    return oracle.load()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(o, pin):
    pin(o)


def test_empty_batch(o):
    import numpy as np
    x, W = oracle_pins._rand_layer(81, d=16, E=4, f=8, k=2, S=1, T=0)
    r = oracle_pins._call(o, x, W, 2, 0.5)
    assert r.y.shape == (0, 16) and r.active.shape == (0, 2, 8)
    assert np.isfinite(r.y).all()
