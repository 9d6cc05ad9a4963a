"""Pins for the oracle's Lloyd-Max codebook (CPU).

The oracle solves the centroid/midpoint fixed point with its own erfc-based
normal functions; these tests check it against (a) Max's 1960 table, (b) the
1-bit closed form, (c) the fixed-point conditions re-evaluated with scipy's
independent normal distribution and adaptive quadrature, (d) the distortion
bound quoted in "We Built a Python Library That Cuts LLM Memory Usage by
80%", section "Test Suite" (read as sqrt(3)·pi/2 · 4^-b).
"""
import math

import numpy as np
import pytest
from scipy import integrate, stats

from conftest import golden_rows
from oracle import codebook as cb


def _table():
    t = {}
    for row in golden_rows("codebook_max1960.txt"):
        t[(int(row[0]), row[1])] = [float(v) for v in row[2:]]
    return t


def test_one_bit_closed_form():
    c, t = cb.lloyd_max_normal(1)
    assert t.tolist() == [0.0]
    assert c[1] == pytest.approx(math.sqrt(2 / math.pi), abs=1e-13)
    assert c[0] == -c[1]
    assert cb.quantizer_mse(c, t) == pytest.approx(1 - 2 / math.pi, abs=1e-13)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_matches_max_1960_table(bits):
    tab = _table()
    c, t = cb.lloyd_max_normal(bits)
    half = len(c) // 2
    np.testing.assert_allclose(c[half:], tab[(bits, "levels")], atol=2e-4)
    np.testing.assert_allclose(t[half - 1:], tab[(bits, "thresholds")], atol=2e-4)
    # The table prints 4 significant digits, and its 4-bit entry (0.009497)
    # sits 0.04% below the exact fixed point (0.0095010, confirmed by
    # quadrature below): compare to 0.1%.
    assert cb.quantizer_mse(c, t) == pytest.approx(tab[(bits, "mse")][0], rel=1e-3)


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5])
def test_fixed_point_with_independent_normal(bits):
    c, t = cb.lloyd_max_normal(bits)
    edges = np.concatenate(([-np.inf], t, [np.inf]))
    n = stats.norm()
    for j in range(len(c)):
        a, b = edges[j], edges[j + 1]
        mass = n.cdf(b) - n.cdf(a) if b <= 0 else n.sf(a) - n.sf(b)
        first = n.pdf(a) - n.pdf(b)      # integral of x·phi over (a, b)
        assert abs(c[j] - first / mass) < 1e-9, (bits, j)
    np.testing.assert_allclose(t, 0.5 * (c[:-1] + c[1:]), atol=1e-12)
    # symmetric and ascending
    np.testing.assert_array_equal(c, -c[::-1])
    assert np.all(np.diff(c) > 0) and np.all(np.diff(t) > 0)
    assert np.all((t > c[:-1]) & (t < c[1:]))


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_mse_by_quadrature(bits):
    c, t = cb.lloyd_max_normal(bits)
    edges = np.concatenate(([-np.inf], t, [np.inf]))
    total = 0.0
    for j in range(len(c)):
        v, _ = integrate.quad(lambda x: (x - c[j]) ** 2 * stats.norm.pdf(x),
                              edges[j], edges[j + 1], epsabs=1e-15, epsrel=1e-12)
        total += v
    assert cb.quantizer_mse(c, t) == pytest.approx(total, abs=1e-12)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_distortion_bound(bits):
    c, t = cb.lloyd_max_normal(bits)
    assert cb.quantizer_mse(c, t) <= math.sqrt(3) * math.pi / 2 * 4.0 ** -bits


@pytest.mark.parametrize("bits", [2, 4])
def test_local_optimality(bits):
    """Moving any threshold or level away from the solution raises the MSE."""
    c, t = cb.lloyd_max_normal(bits)
    base = cb.quantizer_mse(c, t)
    for j in range(len(t)):
        for eps in (-1e-3, 1e-3):
            t2 = t.copy()
            t2[j] += eps
            assert cb.quantizer_mse(c, t2) > base
    for j in range(len(c)):
        for eps in (-1e-3, 1e-3):
            c2 = c.copy()
            c2[j] += eps
            assert cb.quantizer_mse(c2, t) > base
