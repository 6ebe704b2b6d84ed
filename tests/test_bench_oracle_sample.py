"""Host logic of bench.py's oracle timing sample: the two-point line used to extrapolate the
oracle's H and sweep timings to a whole layer (no GPU, no oracle run)."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


def _fit():
    import bench
    return bench.OracleSample._fit


def test_line_through_two_points_extrapolates():
    fit = _fit()
    # t(x) = 2 + 0.5 x: a fixed part and a part linear in the count
    assert fit(16, 10.0, 64, 34.0, 8192) == pytest.approx(2.0 + 0.5 * 8192)
    assert fit(256, 2.0 + 0.5 * 256, 1024, 2.0 + 0.5 * 1024, 131072) == pytest.approx(
        2.0 + 0.5 * 131072)


def test_negative_slope_counts_as_flat():
    fit = _fit()
    # timing noise can make the larger sample faster: the extrapolation then stays at that time
    assert fit(16, 1.2, 64, 1.0, 8192) == pytest.approx(1.0)


def test_equal_sizes_scale_proportionally():
    fit = _fit()
    # a workload smaller than both samples (both clipped to it): plain proportional scaling
    assert fit(300, 3.0, 300, 3.0, 300) == pytest.approx(3.0)
    assert fit(300, 3.0, 300, 3.0, 600) == pytest.approx(6.0)
