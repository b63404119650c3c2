"""Regression pin: the oracle still reproduces its recorded integer outputs on the
1024-token workload (tests/golden/tiny_seed0.txt, written by make_tiny_golden.py)."""
import os
import sys

import numpy as np

HERE = os.path.join(os.path.dirname(__file__), "golden")
sys.path.insert(0, HERE)
import make_tiny_golden  # noqa: E402


def test_tiny_oracle_matches_recorded_outputs():
    want = {}
    for line in open(os.path.join(HERE, "tiny_seed0.txt")):
        if line.startswith("#"):
            continue
        name, vals = line.split(":")
        want[name] = np.array([int(x) for x in vals.split()])
    got = dict(make_tiny_golden.rows())
    assert set(got) == set(want)
    for name in want:
        np.testing.assert_array_equal(np.asarray(got[name]), want[name], err_msg=name)
