"""The excused-mismatch rule of the parity tests (host only).

Integer outputs may differ from the oracle only where the oracle's own
sampling or accept margin is below 1e-5; those excused mismatches must stay
at or under 0.1% of the decisions as a point rate, with no allowance for the
count's sampling noise.
"""
from tests.parity import RATE, Tally, within_rate


def test_point_rate_cap():
    assert RATE == 1e-3
    assert within_rate(0, 1)
    assert not within_rate(1, 999)        # one near-tie in under 1,000 decisions is over 0.1%
    assert within_rate(1, 1000)
    assert not within_rate(2, 1194)       # 0.17% fails
    assert within_rate(10, 10000)
    assert not within_rate(11, 10000)


def test_tally_pools_by_kind():
    a, b = Tally(), Tally()
    a.count("draft", 1500, 1)
    b.count("draft", 500, 0)
    b.count("final", 100, 1)
    a.add(b)
    assert (a.decisions, a.excused) == (2100, 2)
    assert a.by_kind == {"draft": [2000, 1], "final": [100, 1]}
    a.check()
    a.count("final", 0, 1)                # 3 of 2100: over the cap
    try:
        a.check()
    except AssertionError:
        pass
    else:
        raise AssertionError("3 excused of 2100 decisions must fail")
