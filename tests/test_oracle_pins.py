"""The CPU oracle against its pins (no GPU)."""
import time

import numpy as np
import pytest

import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_tiny_config_oracle_is_fast(orc):
    """The tiny layer (hidden 256, 16 experts, top-2, intermediate 128) runs well under 1 s."""
    ly = P.make_tiny_layer(orc)
    x = np.random.default_rng(0).standard_normal(256)
    t = time.perf_counter()
    orc.layer(ly, x, x)
    assert time.perf_counter() - t < 1.0
