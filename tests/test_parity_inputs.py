"""The parity inputs do what the GPU tests say they do (no GPU needed).

The wide-logit-range cases of the calibration tests claim that rows raise the kernels' lazy
reference max mid-walk (block_mass raises only above 64 log2 units, dense_fwd_mass above
16), that later blocks underflow against the first, and that the two column halves of a
row end far apart.  These checks hold the seeded data to those claims, so a change of the
generator cannot silently turn the cases into easy ones.
"""
import numpy as np
import pytest

import helpers as Hp

WLS = Hp.small_workloads()
CASES = [WLS[0], WLS[1], WLS[3]]


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_wide_range_keys_spreads(wl):
    q, k, _ = Hp.draw(wl, value_scale=1.0, sharp=1.0)
    spreads = {}
    for ramp in ("ascending", "descending", "odd_blocks"):
        _, _, scale, bmax = Hp.wide_range_keys(wl, q, k, ramp)
        assert scale > 0
        row_max = bmax.max(-1)
        # the median valid row's max logit sits at the requested 85 log2 units
        assert abs(np.median(row_max) - 85.0) < 1e-6
        spreads[ramp] = bmax
    a = spreads["ascending"]
    # block_mass's halves: a half's first block vs the rest of that half (> 64 log2 units)
    assert np.median(a[..., 0::2].max(-1) - a[..., 0]) > 64.0
    assert np.median(a[..., 1::2].max(-1) - a[..., 1]) > 64.0
    # dense_fwd_mass's first step (blocks 0 and 1) vs the rest (> 16 log2 units)
    assert np.median(a[..., 2:].max(-1) - a[..., :2].max(-1)) > 16.0
    d = spreads["descending"]
    # later blocks lie far below the first: their exponentials underflow against it
    assert np.median(d[..., :2].max(-1) - d[..., -2:].max(-1)) > 40.0
    o = spreads["odd_blocks"]
    # the odd half's reference max ends far above the even half's
    assert np.median(o[..., 1::2].max(-1) - o[..., 0::2].max(-1)) > 64.0
