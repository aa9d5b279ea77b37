"""Host logic of the profile builder: verify-length splits and the table."""
import numpy as np
import pytest


def test_split_lengths():
    from speculative_decoding_semi_b200.profile import split_lengths
    for B, K in ((1, 1), (5, 3), (64, 8)):
        for n in (B, B + 1, B * (K + 1) - 1, B * (K + 1)):
            L = split_lengths(n, B, K)
            assert int((L + 1).sum()) == n and L.min() >= 0 and L.max() <= K
            assert L.max() - L.min() <= 1
    with pytest.raises(ValueError):
        split_lengths(3, 4, 2)
    with pytest.raises(ValueError):
        split_lengths(13, 4, 2)


def test_interpolate():
    from speculative_decoding_semi_b200.profile import grid_points, interpolate
    t = interpolate(np.array([4, 8, 12]), np.array([1.0, 1.2, 1.8]), 16)
    assert t.shape == (16,)
    assert t[0] == t[3] == np.float32(1.0)          # below the grid: the first value
    assert abs(t[5] - 1.1) < 1e-6                   # n = 6: halfway between 4 and 8
    assert abs(t[15] - (1.8 + 0.15 * 4)) < 1e-6     # beyond: the last slope, 0.6 / 4 per token
    # noise that would make T decrease is flattened
    t = interpolate(np.array([1, 2, 3]), np.array([1.0, 0.9, 1.5]), 3)
    assert np.all(np.diff(t) >= 0)
    g = grid_points(64, 8, 8)
    assert g[0] == 64 and g[-1] == 576 and np.all(np.diff(g) > 0)
