"""The oracle against its pins (CPU only).  See oracle_pins.py for what each
pin checks and why it is independent of the oracle's own code."""
import pytest

import oracle
import oracle_pins


@pytest.fixture(scope="module")
def o():
    return oracle.default()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(o, pin):
    pin(o)


def test_thread_count_does_not_change_results():
    import numpy as np
    r = np.random.Generator(np.random.PCG64(9))
    X, Wg, Wu = r.standard_normal((7, 33)), r.standard_normal((21, 33)), r.standard_normal((21, 33))
    o = oracle.default()
    o.set_num_threads(1)
    a = o.swiglu_fwd_f64(X, Wg, Wu)["H"]
    o.set_num_threads(0)
    b = o.swiglu_fwd_f64(X, Wg, Wu)["H"]
    assert np.array_equal(a, b)
