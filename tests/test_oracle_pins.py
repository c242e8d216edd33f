"""The fp64 oracle against facts fixed by the pages and by mathematics (CPU only)."""
import numpy as np
import pytest

import oracle
import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, oracle_lib):
    pin(oracle_lib)


def test_threads_do_not_change_results(oracle_lib):
    rng = np.random.default_rng(8)
    q, k = rng.standard_normal((2, 2, 2, 11, 6))
    v = rng.standard_normal((2, 2, 11, 5))
    beta = rng.uniform(0, 1, (2, 2, 11))
    o1, S1 = oracle.fwd(q, k, v, beta, threads=1, lib=oracle_lib)
    o4, S4 = oracle.fwd(q, k, v, beta, threads=4, lib=oracle_lib)
    assert np.array_equal(o1, o4) and np.array_equal(S1, S4)


def test_golden_regression(oracle_lib):
    """Stored oracle outputs (tests/golden/make_golden.py) guard against silent edits."""
    import golden_cases
    for case in golden_cases.load_all():
        o, ST = oracle.fwd(case["q"], case["k"], case["v"], case["beta"], case["S0"],
                           threads=1, lib=oracle_lib)
        np.testing.assert_allclose(o, case["o"], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(ST, case["S_T"], rtol=1e-13, atol=1e-13)
