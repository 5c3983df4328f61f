"""The method page's cost claim ("Verification", and the log-log slope of its operation
proxy): at bounded degree the hybrid layer's work grows linearly in N.  Timed on the
GPU at fixed in-degree 8 (+ self-loop), r = 16: the log-log slope of the forward time
over N = 2^18 .. 2^21 lies near 1 (loose bounds: a shared GPU adds timing noise, and the
fixed per-launch cost flattens the slope at the small end)."""
import pytest

import bench

pytestmark = pytest.mark.gpu


def test_forward_time_grows_linearly_in_n():
    pts = bench.sweep_points(range(18, 22), steps=15)
    slope = bench.loglog_slope(pts)
    assert 0.8 <= slope <= 1.15, (slope, pts)
    # and the time per edge does not grow with N
    per_edge = [ms / e for _, e, ms in pts]
    assert per_edge[-1] <= 1.25 * per_edge[0], pts
