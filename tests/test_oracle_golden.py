"""The f64 oracle reproduces its stored outputs on tiny seeded problems
(tests/golden/oracle_tiny.json, written by tests/golden/make_golden.py from
the oracle alone): a guard against accidental changes to the oracle.  CPU only."""
import json
import os
import sys

import numpy as np

sys.path.insert(0, os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden"))
import make_golden  # noqa: E402


def test_oracle_matches_stored_outputs():
    with open(make_golden.OUT) as f:
        stored = json.load(f)
    now = make_golden.cases()
    assert sorted(stored) == sorted(now)
    for name, outs in stored.items():
        for k, rec in outs.items():
            got = np.asarray(now[name][k], dtype=np.float64)
            assert list(got.shape) == rec["shape"], (name, k)
            np.testing.assert_allclose(got.ravel(), np.asarray(rec["values"]), rtol=1e-12,
                                       atol=1e-14, err_msg=f"{name}.{k}")
