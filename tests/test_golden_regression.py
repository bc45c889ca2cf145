"""The oracle still reproduces its recorded outputs (tests/golden/oracle_small.json)."""
import json
import os

import numpy as np

from tests.golden.make_golden import compute

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_matches_recorded_golden():
    with open(os.path.join(HERE, "oracle_small.json")) as f:
        want = json.load(f)
    got = compute()
    for name, case in want.items():
        for hw, hg in zip(case["heads"], got[name]["heads"]):
            assert hw["kept"] == hg["kept"]
            for key in ("I", "r", "Z"):
                np.testing.assert_allclose(hg[key], hw[key], rtol=1e-12, atol=1e-16)
