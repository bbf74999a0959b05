"""The oracle against its stored results on the tiny configuration (no GPU).

tests/golden/tiny_oracle.json is written by tests/golden/make_golden.py, which calls only the
oracle and the seeded input generator (the pages print no worked example with numbers).
A mismatch means the oracle's arithmetic changed: rerun the script only when a change is
deliberate, and justify it by the passage it follows.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))

import make_golden  # noqa: E402


def test_oracle_matches_its_stored_tiny_results():
    with open(os.path.join(HERE, "golden", "tiny_oracle.json")) as f:
        want = json.load(f)
    got = make_golden.compute()
    assert got["workload"] == want["workload"] and got["mass_shape"] == want["mass_shape"]
    np.testing.assert_allclose(got["mass"], want["mass"], rtol=0, atol=1e-12)
    # every row of masses is a distribution
    m = np.asarray(got["mass"]).reshape(-1, want["mass_shape"][-1])
    assert np.allclose(m.sum(1), 1.0, atol=1e-12)
    assert got["selections"] == want["selections"]
    a, b = got["attention_0.99"], want["attention_0.99"]
    assert abs(a["sum"] - b["sum"]) <= 1e-9 * max(1.0, abs(b["sum"]))
    assert abs(a["sum_sq"] - b["sum_sq"]) <= 1e-9 * max(1.0, abs(b["sum_sq"]))
    np.testing.assert_allclose(a["row0"], b["row0"], rtol=0, atol=1e-12)
    assert abs(a["lse_finite_sum"] - b["lse_finite_sum"]) <= 1e-9 * max(1.0, abs(b["lse_finite_sum"]))
    # the selections grow with the threshold, and only the lower thresholds drop blocks
    sizes = [len(want["selections"][t]["col_idx"]) for t in sorted(want["selections"], key=float)]
    assert sizes == sorted(sizes) and sizes[0] < sizes[-1]
