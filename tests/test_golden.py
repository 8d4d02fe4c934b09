"""The oracle against its frozen regression record (CPU only)."""
import json
import os

import numpy as np

from tests.golden import make_golden


def test_oracle_matches_golden_record():
    path = os.path.join(os.path.dirname(make_golden.__file__), "oracle_small_case.json")
    with open(path) as f:
        rec = json.load(f)
    out, yf, yb = make_golden.compute()
    for key, arr in (("out", out), ("y_fwd", yf), ("y_rev", yb)):
        want = np.array([float.fromhex(v) for v in rec[key]])
        got = arr.ravel()
        # libm exp/log1p may differ by an ulp across hosts; the arithmetic may not.
        assert np.max(np.abs(got - want)) <= 1e-13 * np.max(np.abs(want)), key
