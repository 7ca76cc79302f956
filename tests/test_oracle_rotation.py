"""Pins of the oracle's randomized Hadamard transform (CPU only).

What is pinned, and against what:
* SplitMix64 -- the published known-answer vector (golden fixture).
* Hadamard order -- Sylvester's recursive construction H_2n = [[H, H], [H, -H]].
* FWHT -- equals multiplication by that matrix, exactly on +-1 data.
* closed form -- x = s1 gives D1 x = 1, so u = H 1 = d e_0 exactly (pins the
  sign application and the normalization).
* R orthonormal, R^-1 R = I, inner products preserved (the pages' reason for
  using a rotation: "an orthogonal rotation preserves inner products").
"""
import math

import numpy as np
import pytest

import oracle as o


def test_splitmix64_known_answer(golden):
    rows = golden("splitmix64_seed1234567.txt")
    assert rows[0][0] == "seed"
    seed = int(rows[0][1])
    expected = [int(r[0]) for r in rows[1:]]
    assert o.splitmix64(seed, len(expected)) == expected


def test_rotation_signs_are_top_bits():
    outs = o.splitmix64(0, 16)
    s = o.rotation_signs(0, 16)
    assert s.dtype == np.int8
    assert set(np.unique(s)) <= {-1, 1}
    assert list(s) == [(-1 if w >= 2**63 else 1) for w in outs]
    s2 = o.rotation_signs(0, 16, second=True)
    assert list(s2) == [(-1 if w >= 2**63 else 1)
                        for w in o.splitmix64(0x9E3779B97F4A7C15, 16)]
    assert not np.array_equal(s, s2)


def test_rotation_signs_balanced():
    s = o.rotation_signs(7, 4096)
    assert abs(int(s.sum())) < 4 * math.sqrt(4096)


def _sylvester(d):
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


@pytest.mark.parametrize("d", [1, 2, 4, 8, 64, 128, 256])
def test_hadamard_matrix_is_sylvester(d):
    assert np.array_equal(o.hadamard_matrix(d), _sylvester(d))


@pytest.mark.parametrize("d", [8, 64, 128, 256])
def test_fwht_matches_matrix(d):
    h = _sylvester(d)
    eye = np.eye(d, dtype=np.float32)
    # columns of H, exactly, in float32
    assert np.array_equal(o.fwht(eye), h.T.astype(np.float32))
    rng = np.random.default_rng(d)
    x = rng.integers(-3, 4, size=(5, d)).astype(np.float32)   # small ints: exact
    assert np.array_equal(o.fwht(x), (x.astype(np.float64) @ h.T).astype(np.float32))
    xf = rng.standard_normal((5, d))
    np.testing.assert_allclose(o.fwht(xf, np.float64), xf @ h.T, rtol=0, atol=1e-12)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("seed", [0, 1, 12345])
def test_signs_closed_form(d, seed):
    s1 = o.rotation_signs(seed, d)
    u = o.fwht(np.where(s1 < 0, -s1.astype(np.float32), s1.astype(np.float32)))
    expect = np.zeros(d, np.float32)
    expect[0] = d
    assert np.array_equal(u, expect)
    # the same through the orthonormal float64 route: R s1 = sqrt(d) e_0
    r = o.rht_forward(s1.astype(np.float64), s1)
    assert abs(r[0] - math.sqrt(d)) < 1e-12 and np.abs(r[1:]).max() < 1e-12


@pytest.mark.parametrize("d", [64, 128, 256])
def test_rotation_orthonormal_and_inverse(d):
    s1 = o.rotation_signs(3, d)
    eye = np.eye(d)
    rot = o.rht_forward(eye, s1)              # rows: R e_j
    np.testing.assert_allclose(rot @ rot.T, eye, atol=1e-12)
    # float32 butterflies, normalized afterwards: R R^T = I to 1e-6
    r32 = o.fwht(np.where(s1 < 0, -eye, eye).astype(np.float32)).astype(np.float64) / math.sqrt(d)
    np.testing.assert_allclose(r32 @ r32.T, eye, atol=1e-6)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((4, d))
    np.testing.assert_allclose(o.rht_inverse(o.rht_forward(x, s1), s1), x, atol=1e-12)
    # R as an explicit matrix agrees with the transform
    rmat = _sylvester(d) * s1[None, :] / math.sqrt(d)
    np.testing.assert_allclose(o.rht_forward(x, s1), x @ rmat.T, atol=1e-12)


def test_inner_products_preserved():
    d = 128
    rng = np.random.default_rng(5)
    q = rng.standard_normal((16, d))
    k = rng.standard_normal((16, d)) * 3
    s1 = o.rotation_signs(11, d)
    lhs = np.sum(o.rht_forward(q, s1) * o.rht_forward(k, s1), axis=1)
    rhs = np.sum(q * k, axis=1)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-5, atol=1e-9)


def test_pairwise_sum_order():
    # tree order: (a0 + a1) + (a2 + a3); a left-to-right sum gives 1 here
    x = np.array([1e8, 1.0, -1e8, 1.0], np.float32)
    assert o.pairwise_sum_f32(x) == np.float32(0.0)
    rng = np.random.default_rng(2)
    y = rng.standard_normal((3, 256)).astype(np.float32)
    np.testing.assert_allclose(o.pairwise_sum_f32(y), y.astype(np.float64).sum(1), rtol=1e-5)
