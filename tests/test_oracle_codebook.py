"""Pins of the oracle's Lloyd-Max codebook (CPU only).

* Max (1960), Table I -- published output levels and distortions (golden).
* Lloyd-Max optimality -- every centroid is its cell's conditional mean
  (checked by numerical integration with scipy, not by the oracle's closed form)
  and every boundary is the midpoint of its neighbours.
* 1-bit closed form c = +-sqrt(2/pi); uniqueness for a log-concave density (two
  different starts converge to the same table).
* float32 table: exact odd symmetry, middle boundary exactly 0, boundaries are
  the float32 midpoints.
"""
import math

import numpy as np
import pytest
from scipy import integrate

import oracle as o


def _max_table(golden):
    out = {}
    for row in golden("max1960_gaussian.txt"):
        bits = int(row[0])
        out[bits] = (float(row[1]), [float(v) for v in row[2:]])
    return out


def _distortion(c):
    """E[(X - Q(X))^2] for X ~ N(0,1), by quadrature over each cell."""
    c = np.asarray(c, np.float64)
    edges = [-np.inf] + [(c[j] + c[j + 1]) / 2 for j in range(len(c) - 1)] + [np.inf]
    pdf = lambda x: math.exp(-x * x / 2) / math.sqrt(2 * math.pi)
    tot = 0.0
    for j in range(len(c)):
        val, _ = integrate.quad(lambda x: (x - c[j]) ** 2 * pdf(x), edges[j], edges[j + 1],
                                epsabs=1e-13, epsrel=1e-12)
        tot += val
    return tot


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_matches_max_1960(golden, bits):
    dist, levels = _max_table(golden)[bits]
    c, _ = o.lloyd_max_gaussian(1 << bits)
    pos = c[len(c) // 2:]
    np.testing.assert_allclose(pos, levels, atol=1.2e-3)
    assert abs(_distortion(c) - dist) <= 2e-3 * dist + 1e-5


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_fixed_point_conditions(bits):
    c, _ = o.lloyd_max_gaussian(1 << bits)
    edges = [-np.inf] + [(c[j] + c[j + 1]) / 2 for j in range(len(c) - 1)] + [np.inf]
    pdf = lambda x: math.exp(-x * x / 2) / math.sqrt(2 * math.pi)
    for j in range(len(c)):
        a, b = edges[j], edges[j + 1]
        mass, _ = integrate.quad(pdf, a, b, epsabs=1e-14, epsrel=1e-13)
        first, _ = integrate.quad(lambda x: x * pdf(x), a, b, epsabs=1e-14, epsrel=1e-13)
        assert abs(first / mass - c[j]) < 1e-9
    assert np.all(np.diff(c) > 0)


def test_one_bit_closed_form():
    c, _ = o.lloyd_max_gaussian(2)
    np.testing.assert_allclose(c, [-math.sqrt(2 / math.pi), math.sqrt(2 / math.pi)], atol=1e-14)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_unique_from_two_starts(bits):
    L = 1 << bits
    a, _ = o.lloyd_max_gaussian(L)
    b, _ = o.lloyd_max_gaussian(L, init=np.linspace(-0.1, 0.1, L) + 0.05 * np.arange(L) ** 2)
    np.testing.assert_allclose(a, b, atol=1e-11)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_float32_table(bits):
    cent, bnd = o.codebook(bits)
    L = 1 << bits
    assert cent.dtype == np.float32 and bnd.dtype == np.float32
    assert cent.shape == (L,) and bnd.shape == (L - 1,)
    assert np.array_equal(cent[::-1], -cent)
    assert bnd[L // 2 - 1] == 0.0
    assert np.all(np.diff(bnd) > 0)
    assert np.all(bnd > cent[:-1]) and np.all(bnd < cent[1:])
    mid = ((cent[:-1].astype(np.float32) + cent[1:]) * np.float32(0.5)).astype(np.float32)
    assert np.array_equal(bnd, mid)
    c64, _ = o.lloyd_max_gaussian(L)
    np.testing.assert_allclose(cent, c64, rtol=1e-7, atol=0)
