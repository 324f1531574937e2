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


def test_group_size_rule(osc):
    """The per-layer group size (§6, dynamic group size; the rule is a stated reading): the
    largest G whose density is above 60 %, else G = 32 with its own tier, 0 for the MXFP8
    fallback. Boundaries of the tiers apply as in osc_select_tier (60 % itself is not high)."""
    nan = float("nan")
    assert osc.osc_select_group_size(0.36, 0.703, 0.726) == (64, 2)      # QKV-like: high at 32 and 64
    assert osc.osc_select_group_size(0.90, 0.70, 0.50) == (32, 2)        # high at 16 and 32 only
    assert osc.osc_select_group_size(0.65, 0.50, 0.40) == (16, 2)        # high only at the finest G
    assert osc.osc_select_group_size(0.40, 0.60, 0.45) == (32, 1)        # nothing high: G = 32, mid tier
    assert osc.osc_select_group_size(0.17, 0.27, 0.37) == (0, 0)         # W2-like: G = 32 falls back to MXFP8
    assert osc.osc_select_group_size(0.20, 0.3499, 0.5999) == (0, 0)
    assert osc.osc_select_group_size(0.20, 0.35, 0.30) == (32, 1)        # 35 % is the middle tier
    assert osc.osc_select_group_size(nan, nan, nan) == (64, 2)           # no events anywhere
    assert osc.osc_select_group_size(0.5, 0.5, 0.6000001) == (64, 2)


def test_group_size_on_the_oracle_densities(osc, oracle):
    """On the synthetic module inputs the rule picks G = 64 for the attention input (its
    density stays above 60 % at G = 32 and 64) and the MXFP8 fallback for W2 (every G below
    60 %, and G = 32 in the fallback tier), computed from the oracle's own counts."""
    def cbar(case, G):
        L = oracle.build_table(case.calib, G)
        nh, nt = oracle.density(case.X, G, L)
        return osc.osc_select_tier(nh.astype(np.int32), nt.astype(np.int32))[1]
    q = I.qkv_case(256, calib_tokens=512)
    assert osc.osc_select_group_size(*(cbar(q, G) for G in (16, 32, 64)))[0] == 64
    w = I.w2_case(M=256, calib_tokens=512)
    assert osc.osc_select_group_size(*(cbar(w, G) for G in (16, 32, 64))) == (0, 0)
