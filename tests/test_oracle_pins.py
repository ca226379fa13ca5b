"""The oracle against facts fixed outside itself (CPU only)."""
import pytest

import oracle
from tests import oracle_pins


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(oracle)


def test_compare_bounds():
    import numpy as np
    ref = np.array([0.0, 1.0, 100.0])
    assert oracle.compare(ref + np.array([0.009, 0.019, 0.0]), ref)["nfail"] == 0
    assert oracle.compare(ref + np.array([0.011, 0.0, 0.0]), ref)["nfail"] == 1
    assert oracle.compare(ref + np.array([0.0, 0.021, 0.0]), ref)["nfail"] == 1
    assert not oracle.compare(ref * 1.01, ref)["ok"]   # normwise 1e-2 > 5e-3
