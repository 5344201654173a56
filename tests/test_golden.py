"""Regression guard: the oracle still reproduces its stored tiny case.

tests/golden/tiny_oracle.npz was written by tests/golden/make_golden.py,
which calls only the oracle and the seeded generators.
"""
import os

import numpy as np

from tests.golden import make_golden


def test_oracle_matches_stored_tiny_case():
    ref = np.load(os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.npz"))
    now = make_golden.compute()
    assert sorted(ref.files) == sorted(now.keys())
    for k in ref.files:
        np.testing.assert_allclose(now[k], ref[k], rtol=1e-12, atol=1e-12, err_msg=k)
