"""The pooled excused-mismatch rule of the parity tests (host only).

Excused mismatches (integer outputs that differ where the oracle's sampling or
accept margin is below 1e-5) must stay under 0.1% of the decisions; the check
treats the count as a Poisson sample and fails when it is significantly above
that rate.
"""
import math

import pytest

from tests.parity import RATE, excused_limit


def _tail(lam, k):
    """P(X >= k) for X ~ Poisson(lam), by direct summation."""
    return 1.0 - sum(math.exp(-lam) * lam ** i / math.factorial(i) for i in range(k))


@pytest.mark.parametrize("n", [50, 400, 1194, 2000, 3500, 10000])
def test_limit_is_the_five_percent_critical_count(n):
    lam = RATE * n
    k = excused_limit(n)
    if k > 2:
        assert _tail(lam, k) < 0.05 <= _tail(lam, k - 1)
    else:
        assert _tail(lam, 2) < 0.05 or k == 2


def test_limit_rejects_a_rate_ten_times_too_high():
    for n in (1194, 2000, 10000):
        assert excused_limit(n) <= 10 * RATE * n


def test_limit_allows_one_near_tie_and_grows_with_the_sample():
    lims = [excused_limit(n) for n in (1, 10, 100, 1000, 10000, 100000)]
    assert lims[0] == 2 and lims == sorted(lims)
