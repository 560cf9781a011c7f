"""The oracle reproduces the stored golden fixtures (tests/golden/, written by
tests/golden/make_golden.py from the oracle itself; the pages print no
numeric worked example).  A failure means the oracle's arithmetic changed."""
import os

import numpy as np
import pytest

from tests.golden import make_golden as mg

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.mark.parametrize("case", mg.cases(), ids=lambda c: c[0])
def test_oracle_matches_golden_fixture(case):
    name, _, arrays = case
    stored = mg.parse(open(os.path.join(HERE, name)).read())
    assert set(stored) == set(arrays)
    for label, a in arrays.items():
        np.testing.assert_allclose(np.atleast_2d(a), stored[label], rtol=1e-13, atol=1e-15,
                                   err_msg=f"{name} [{label}]")
