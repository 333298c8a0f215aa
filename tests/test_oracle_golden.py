"""Regression of the oracle against its committed fixture (no GPU).

The fixture is written by tests/golden/make_golden.py from the oracle alone.
"""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.join(os.path.dirname(__file__), "golden"))
import make_golden  # noqa: E402


def test_oracle_matches_regression_fixture():
    qh, o, lse = make_golden.compute()
    lines = [l.split() for l in open(make_golden.OUT) if not l.startswith("#")]
    rec = {}
    orows = {}
    for parts in lines:
        if parts[0] in ("o", "lse"):
            orows.setdefault(int(parts[1]), {})[parts[0]] = [float(x) for x in parts[2:]]
        else:
            rec[parts[0]] = parts[1:]
    assert np.array_equal(np.float32([float(x) for x in rec["qs"]]), qh["qs"])
    assert np.array_equal(np.float32([float(x) for x in rec["ks"]]), qh["ks"])
    assert np.array_equal(np.float32([float(x) for x in rec["mu"]]), qh["mu"][:8])
    assert np.array_equal(np.float32([float(x) for x in rec["vs"]]), qh["vs"][:8])
    assert int(rec["q8sum"][0]) == int(qh["q8"].astype(np.int64).sum())
    assert int(rec["k8sum"][0]) == int(qh["k8"].astype(np.int64).sum())
    assert int(rec["v8sum"][0]) == int(qh["v8"].astype(np.int64).sum())
    for r, row in enumerate(make_golden.ROWS):
        assert np.allclose(orows[row]["o"], o[r, :8], rtol=1e-8, atol=1e-12)
        assert abs(orows[row]["lse"][0] - lse[r]) < 1e-10


def test_window_oracle_matches_regression_fixture():
    o1, l1, o3, l3 = make_golden.compute_window()
    got = {}
    for parts in (l.split() for l in open(make_golden.OUT_WIN) if not l.startswith("#")):
        got[(parts[0], parts[1], int(parts[2]))] = [float(x) for x in parts[3:]]
    for tag, o, lse in (("s1", o1, l1), ("s3", o3, l3)):
        for r, row in enumerate(make_golden.WIN_ROWS):
            assert np.allclose(got[("o", tag, row)], o[r, :8], rtol=1e-8, atol=1e-12)
            assert abs(got[("lse", tag, row)][0] - lse[r]) < 1e-10
    # the split form differs from the unsplit one by P rounding points only
    assert np.abs(o1 - o3).max() < 0.05 and np.abs(o1 - o3).max() > 0
