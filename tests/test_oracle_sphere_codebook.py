"""Pins of the oracle's unit-sphere codebook (a Lloyd-Max quantizer for the exact
distribution of a rotated, normalized coordinate scaled by sqrt(d)).

Each check is tied to something other than the oracle's own formulas:
numerical quadrature of the density, the closed form of E|y| for a coordinate
of a random unit vector, Monte Carlo over random unit vectors, the optimality
of Lloyd-Max (under the true density it beats the N(0,1) codebook), and the
large-d limit (the N(0,1) codebook).
"""
import math

import numpy as np
import pytest
from scipy.integrate import quad

import oracle as o

DIMS = [64, 128, 256]


def _density(z, d):
    return o.sphere_density(z, d)


@pytest.mark.parametrize("d", DIMS)
def test_density_integrates_to_one(d):
    r = math.sqrt(d)
    total, err = quad(_density, -r, r, args=(d,), epsabs=1e-13, limit=200)
    assert abs(total - 1.0) < 1e-10


@pytest.mark.parametrize("d", DIMS)
def test_mass_and_first_moment_match_quadrature(d):
    for a, b in ((-math.inf, -2.0), (-1.3, 0.4), (0.0, 0.7), (1.1, 2.9), (2.5, math.inf), (-0.2, 0.2)):
        lo, hi = max(a, -math.sqrt(d)), min(b, math.sqrt(d))
        m, _ = quad(_density, lo, hi, args=(d,), epsabs=1e-14, limit=200)
        f, _ = quad(lambda z: z * _density(z, d), lo, hi, epsabs=1e-14, limit=200)
        assert abs(o.sphere_mass(a, b, d) - m) < 1e-11
        assert abs(o.sphere_first_moment(a, b, d) - f) < 1e-11


@pytest.mark.parametrize("d", DIMS)
def test_one_bit_centroid_is_the_mean_absolute_coordinate(d):
    # E|y| for a coordinate y of a uniform unit vector of R^d is
    # Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2)); the 1-bit centroid is sqrt(d) E|y|
    expect = math.sqrt(d) * math.exp(math.lgamma(d / 2) - math.lgamma((d + 1) / 2)) / math.sqrt(math.pi)
    c, _ = o.lloyd_max_sphere(2, d)
    assert abs(c[1] - expect) < 1e-12 and abs(c[0] + expect) < 1e-12


@pytest.mark.parametrize("d", DIMS)
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_fixed_point_conditions(d, bits):
    c, _ = o.lloyd_max_sphere(1 << bits, d)
    r = math.sqrt(d)
    edges = [-r] + [(c[j] + c[j + 1]) / 2 for j in range(len(c) - 1)] + [r]
    for j in range(len(c)):
        m, _ = quad(_density, edges[j], edges[j + 1], args=(d,), epsabs=1e-14, limit=200)
        f, _ = quad(lambda z: z * _density(z, d), edges[j], edges[j + 1], epsabs=1e-14, limit=200)
        assert abs(f / m - c[j]) < 1e-9
    assert np.allclose(c, -c[::-1], rtol=0, atol=1e-12)


def _distortion(cent, d):
    """E (Z - Q(Z))^2 under the sphere density, cell by cell by quadrature."""
    r = math.sqrt(d)
    edges = [-r] + [(cent[j] + cent[j + 1]) / 2 for j in range(len(cent) - 1)] + [r]
    return sum(quad(lambda z: (z - cent[j]) ** 2 * _density(z, d), edges[j], edges[j + 1],
                    epsabs=1e-15, limit=200)[0] for j in range(len(cent)))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_beats_the_gaussian_codebook_under_the_true_density(d, bits):
    cs, _ = o.lloyd_max_sphere(1 << bits, d)
    cg, _ = o.lloyd_max_gaussian(1 << bits)
    ds, dg = _distortion(cs, d), _distortion(cg, d)
    assert ds < dg


def test_tends_to_the_gaussian_codebook():
    gaps = []
    for d in (4096, 16384):
        cs, _ = o.lloyd_max_sphere(16, d, tol=1e-11)
        cg, _ = o.lloyd_max_gaussian(16)
        gaps.append(np.abs(cs - cg).max())
    assert gaps[1] < 5e-4 and gaps[1] < gaps[0] / 3


def test_monte_carlo_on_random_unit_vectors():
    d, n = 128, 40000
    rng = np.random.default_rng(123)
    g = rng.standard_normal((n, d))
    z = (math.sqrt(d) * g[:, 0] / np.linalg.norm(g, axis=1))      # one coordinate per vector
    c1, _ = o.lloyd_max_sphere(2, d)
    a = np.abs(z)
    assert abs(a.mean() - c1[1]) < 4 * a.std() / math.sqrt(n)
    cent, bnd = o.sphere_codebook(3, d)
    q = cent[o.bucket_index(z.astype(np.float32), bnd)].astype(np.float64)
    err = (z - q) ** 2
    assert abs(err.mean() - _distortion(cent.astype(np.float64), d)) < 4 * err.std() / math.sqrt(n)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_float32_tables_are_odd_symmetric(bits):
    cent, bnd = o.sphere_codebook(bits, 128)
    assert cent.dtype == np.float32 and bnd.dtype == np.float32
    assert np.array_equal(cent, -cent[::-1])
    assert bnd[len(bnd) // 2] == 0.0 and np.array_equal(bnd, -bnd[::-1])
    assert np.all(np.diff(cent) > 0)
