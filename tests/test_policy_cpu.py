"""The block-policy rule of the blog's "Calibration-driven block selection" (host logic in
the C library, no GPU): hand-worked cases at and around every threshold of the three tiers."""
import json
import os

import pytest

from fp8_mixed_precision_mxq_b200 import policy

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tier_rule.json")
FIX = json.load(open(GOLDEN))


@pytest.mark.parametrize("tier", ["low", "mid", "high"])
def test_tier_thresholds(tier):
    assert list(policy.thresholds(tier)) == FIX["tiers"][tier]


@pytest.mark.parametrize("case", FIX["cases"], ids=lambda c: "%s-%s-%s" % (c["tier"], c["off"], c["on"]))
def test_rule_cases(case):
    assert policy.select(case["off"], case["on"], case["tier"]) == case["policy"], case["why"]


def test_rule_rejects_nan_and_unknown_tier():
    with pytest.raises(ValueError):
        policy.select(float("nan"), 20.0, "high")
    from fp8_mixed_precision_mxq_b200 import _lib
    assert _lib.lib().mxq_select_policy(20.0, 20.0, 7) == -1


def test_rule_precedence_is_monotone():
    """With a fixed transform gain, raising the SQNR moves a block from bf16 to W4A8 to one
    W4A4 policy (transform_on when the gain exceeds the margin, else plain) and never back."""
    for tier in ("low", "mid", "high"):
        _, _, margin = policy.thresholds(tier)
        for gain in (0.0, 0.3, 0.6, 3.0):
            seq = [policy.select(0.5 * i, 0.5 * i + gain, tier) for i in range(80)]
            final = "transform_on" if gain > margin else "plain_mxfp4"
            allowed = ["bf16", "w4a8", final]
            ranks = [allowed.index(p) for p in seq]
            assert ranks == sorted(ranks) and ranks[-1] == 2, (tier, gain, seq)
