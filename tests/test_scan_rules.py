"""The composition rule the Bi-WKV backward scans with, checked against the
sums it stands for.

For a segment x_0..x_{L-1} and decay a, the forward aggregate is
    A = sum_j a^{L-1-j} x_j,    H = sum_j (L-1-j) a^{L-1-j} x_j,
the decayed sum and its distance-weighted part (the derivative of the decay
sums of eq. 5 with respect to w needs the latter).  Appending a segment of
length L2 with aggregate (A2, H2) gives
    A = a^{L2} A1 + A2,    H = a^{L2} (H1 + L2 A1) + H2,
and this rule is associative, so (A, H) can be scanned across threads, warps
and CTAs in any grouping.  The token walk of the kernel,
    H <- a (H + A),  A <- a A + x_i,
is the same rule with L2 = 1.
"""
import numpy as np
import pytest


def direct(x, a):
    L = len(x)
    d = (L - 1 - np.arange(L)).astype(np.float64)
    return float(np.sum(a ** d * x)), float(np.sum(d * a ** d * x))


def cross(left, a, L2, right):
    A1, H1 = left
    A2, H2 = right
    aL = a ** L2
    return aL * A1 + A2, aL * (H1 + L2 * A1) + H2


def walk(x, a):
    A = H = 0.0
    for xi in x:
        H = a * (H + A)
        A = a * A + xi
    return A, H


@pytest.mark.parametrize("a", [0.3, 0.97, 1.0, 1.04])
def test_token_walk_is_the_segment_sums(a):
    rng = np.random.default_rng(int(a * 100))
    x = rng.normal(size=23)
    np.testing.assert_allclose(walk(x, a), direct(x, a), rtol=1e-12)


@pytest.mark.parametrize("a", [0.5, 0.99, 1.0, 1.02])
def test_appending_a_segment(a):
    rng = np.random.default_rng(int(a * 1000))
    x = rng.normal(size=40)
    for cut in (1, 7, 16, 39):
        got = cross(direct(x[:cut], a), a, len(x) - cut, direct(x[cut:], a))
        np.testing.assert_allclose(got, direct(x, a), rtol=1e-12)


def test_rule_is_associative():
    rng = np.random.default_rng(11)
    a = 0.93
    x = rng.normal(size=30)
    s1, s2, s3 = x[:8], x[8:19], x[19:]
    p1, p2, p3 = direct(s1, a), direct(s2, a), direct(s3, a)
    left_first = cross(cross(p1, a, len(s2), p2), a, len(s3), p3)
    right_first = cross(p1, a, len(s2) + len(s3), cross(p2, a, len(s3), p3))
    np.testing.assert_allclose(left_first, right_first, rtol=1e-12)
    np.testing.assert_allclose(left_first, direct(x, a), rtol=1e-12)
