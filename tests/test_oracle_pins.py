"""The oracle against its pins (CPU only)."""
import pytest

import oracle
import oracle_pins


@pytest.fixture(scope="module")
def o():
    return oracle.get()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(o, pin):
    pin(o)


def test_tolerance_formula():
    """ulp16 of the bound: 2^(floor(log2|v|)-10) for normal binary16 values, 2^-24 below."""
    import numpy as np
    y = np.array([1.0, 1.5, 2.0, 1e-6, 0.0, -3.0])
    X = np.zeros((1, 4), dtype=np.float16)
    tol = oracle.tolerance(y, np.repeat(X, 6, axis=0), 1.0)
    expect = [2.0 ** -10, 2.0 ** -10, 2.0 ** -9, 2.0 ** -24, 2.0 ** -24, 2.0 ** -9]
    assert tol.tolist() == expect
    # the ulp term equals numpy's binary16 spacing for normal values
    for v in (1.0, 3.7, 1000.0, 0.001):
        assert oracle.tolerance(np.array([v]), X, 1.0)[0] == float(np.spacing(np.float16(v)))
    # the 1e-3 * alpha * sum|x| term
    X2 = np.array([[1.0, -2.0, 0.5]], dtype=np.float16)
    assert oracle.tolerance(np.array([[0.0]]), X2, 2.0)[0, 0] == 1e-3 * 2.0 * 3.5 + 2.0 ** -24
