"""The fp64 oracle against its pins (CPU only).  See ``pins.py`` for what fixes
each expected value."""
import pytest

import oracle
from pins import ALL_PINS


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_pin(orc, pin):
    pin(orc)


def test_rejects_short_groups(orc):
    """Maps with a dilation group shorter than k have no valid window."""
    import numpy as np
    x = np.zeros((1, 1, 13, 14, 4))
    with pytest.raises(ValueError):
        orc.forward(x, x, x, None, 7, 2)   # H // d = 6 < k
    with pytest.raises(ValueError):
        orc.axis_window(6, 7, 1, 0)


def test_threads_do_not_change_results(orc):
    import numpy as np
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((3, 2, 9, 10, 4)) for _ in range(3))
    rpb = rng.standard_normal((2, 5, 5))
    a = orc.forward(q, k, v, rpb, 3, 2, nthreads=1)
    b = orc.forward(q, k, v, rpb, 3, 2, nthreads=4)
    assert (a == b).all()
