"""The oracle against its pins (CPU only). Each pin is described in
``oracle_pins.py``; none compares the oracle with itself."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(orc, pin):
    pin(orc)


def test_threads_do_not_change_results(orc):
    import numpy as np
    x = oracle_pins._rows(50, 300, 257, "bf16", 0.5, 2.0)
    w = oracle_pins._rows(51, 1, 257, "bf16", 1.0, 0.1)[0]
    one = orc.layer_norm(x, w, w, 1e-5, nthreads=1)
    many = orc.layer_norm(x, w, w, 1e-5, nthreads=4)
    assert np.array_equal(one, many)
