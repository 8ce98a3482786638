"""The oracle still reproduces the frozen outputs in tests/golden/oracle_regress.npz
(written by tests/golden/make_golden.py, which calls only the oracle)."""
import os

import numpy as np

from golden import make_golden


def test_oracle_matches_frozen_outputs():
    frozen = np.load(os.path.join(os.path.dirname(__file__), "golden", "oracle_regress.npz"))
    now = make_golden.make()
    for k in frozen.files:
        np.testing.assert_array_equal(now[k], frozen[k], err_msg=k)
