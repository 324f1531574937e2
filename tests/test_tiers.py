"""Tier selection of the OSC page (§2.3): the host rule of osc_select_tier on density counts.
It is checked against the tier thresholds of the page's Table 1 text (tests/golden), at and
around the boundaries, and against the oracle's density of the synthetic module inputs.
Host logic only, so no GPU is needed."""
import os

import numpy as np
import pytest

from w4a4_outlier_separated_b200 import inputs as I

GOLD = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def osc():
    from w4a4_outlier_separated_b200 import build
    build.build()
    from w4a4_outlier_separated_b200 import osc as m
    m.lib()
    return m


def _bands():
    out = {}
    for line in open(os.path.join(GOLD, "table1_density_bands.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            f = line.split()
            out[f[0]] = tuple(map(float, f[1:]))
    return out


def test_tier_boundaries_follow_the_page(osc):
    b = _bands()
    high, fp8 = b["tier_high"][0], b["tier_fp8"][0]
    assert (high, fp8) == (0.60, 0.35)
    # one group each: C exactly at a boundary belongs to the middle tier
    assert osc.osc_select_tier([3], [5]) == (1, 3 / 5)                  # C = 60 %: not above 60 %
    assert osc.osc_select_tier([61], [100])[0] == 2
    assert osc.osc_select_tier([7], [20]) == (1, 7 / 20)                # C = 35 %: not below 35 %
    assert osc.osc_select_tier([34], [100])[0] == 0
    assert osc.osc_select_tier([0], [9]) == (0, 0.0)
    assert osc.osc_select_tier([9], [9]) == (2, 1.0)


def test_mean_skips_groups_without_events(osc):
    tier, c = osc.osc_select_tier([1, 0, 3, 0], [2, 0, 4, 0])          # (1/2 + 3/4) / 2
    assert tier == 2 and c == pytest.approx(0.625, abs=0)
    tier, c = osc.osc_select_tier([0, 0, 0], [0, 0, 0])
    assert tier == 2 and np.isnan(c)                                     # nothing escapes the table
    assert osc.osc_select_tier([], []) [0] == 2


def test_bad_counts_are_rejected(osc):
    from w4a4_outlier_separated_b200.osc import OSCError
    with pytest.raises(OSCError):
        osc.osc_select_tier([3], [2])                                    # more hits than events
    with pytest.raises(OSCError):
        osc.osc_select_tier([-1], [2])
    with pytest.raises(ValueError):
        osc.osc_select_tier([1, 2], [3])


def test_module_inputs_land_in_the_page_tiers(osc, oracle):
    """The oracle's density of the synthetic inputs, through the host rule: the attention input
    (fixed channels in 70 % of groups) selects static protection, W2 (diffuse outliers) the
    MXFP8 fallback, as Table 1 places these modules."""
    q = I.qkv_case(512)
    L = oracle.build_table(q.calib, 32)
    nh, nt = oracle.density(q.X, 32, L)
    tier, c = osc.osc_select_tier(nh, nt)
    assert tier == 2 and c > 0.6
    w = I.w2_case(M=512, calib_tokens=1536)
    Lw = oracle.build_table(w.calib, 32)
    nh, nt = oracle.density(w.X, 32, Lw)
    tier, c = osc.osc_select_tier(nh, nt)
    lo, hi = _bands()["w2"]
    assert tier == 0 and lo <= c <= hi
