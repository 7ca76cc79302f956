"""Pins of the oracle's codec: quantizer, packing, norms, QJL sketch (CPU only).

* nearest centroid by brute force in float64 (the boundary count must pick it
  wherever z is not within one float32 ulp of a boundary);
* all-centroid inputs reproduce their indices; ties go to the lower index;
* packing equals the integer sum_i idx_i << (b*i), little-endian;
* closed forms: the zero vector; x = a*s1 (all energy on channel 0);
* empirical distortion ~ Max's D_b on Gaussian and on outlier-channel data;
* QJL: rho = ||Rk - k_hat||; the estimator is unbiased over random rotations
  where MSE-only scoring under-counts by about cos * D_b (the pages report a
  bias of roughly -0.05 for correlated pairs that QJL removes), and its
  variance stays within the Gaussian-sketch figure.
"""
import math

import numpy as np
import pytest

import oracle as o

MAX_D = {2: 0.1175, 3: 0.03455, 4: 0.009497}


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_bucket_is_nearest_centroid(bits):
    cent, bnd = o.codebook(bits)
    rng = np.random.default_rng(bits)
    z = (rng.standard_normal(200_000) * 1.3).astype(np.float32)
    idx = o.bucket_index(z, bnd)
    brute = np.argmin(np.abs(z.astype(np.float64)[:, None] - cent.astype(np.float64)[None, :]), axis=1)
    near = np.min(np.abs(z[:, None].astype(np.float64) - bnd[None, :].astype(np.float64)), axis=1) \
        <= np.spacing(np.abs(z)).astype(np.float64)
    assert np.all((idx == brute) | near)
    # values within one ulp of a boundary are rare (about 1e-6 of the draws)
    assert int(near.sum()) <= 3


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_centroids_round_trip_and_ties(bits):
    cent, bnd = o.codebook(bits)
    assert list(o.bucket_index(cent, bnd)) == list(range(1 << bits))
    # a value exactly on a boundary takes the lower index
    assert list(o.bucket_index(bnd, bnd)) == list(range((1 << bits) - 1))
    assert o.bucket_index(np.float32(-0.0), bnd) == (1 << bits) // 2 - 1


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("d", [8, 64, 128, 256])
def test_pack_is_little_endian_stream(bits, d):
    rng = np.random.default_rng(d + bits)
    idx = rng.integers(0, 1 << bits, size=(7, d))
    packed = o.pack_codes(idx, bits)
    assert packed.shape == (7, bits * d // 8) and packed.dtype == np.uint8
    for n in range(7):
        as_int = sum(int(idx[n, i]) << (bits * i) for i in range(d))
        assert int.from_bytes(packed[n].tobytes(), "little") == as_int
    assert np.array_equal(o.unpack_codes(packed, bits, d), idx)


def test_pack_hand_example():
    # 3-bit codes 5,3,7,0,1,6,2,4 -> bits 101 110 111 000 100 011 010 001 (LSB first)
    packed = o.pack_codes(np.array([[5, 3, 7, 0, 1, 6, 2, 4]]), 3)
    assert list(packed[0]) == [0b11011101, 0b00010001, 0b10001011]


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_zero_vector(bits):
    d = 128
    cent, bnd = o.codebook(bits)
    s1, s2 = o.rotation_signs(0, d), o.rotation_signs(0, d, second=True)
    e = o.encode(np.zeros((1, d), np.float32), s1, cent, bnd, bits, s2)
    assert e["norm16"][0] == 0 and e["rnorm16"][0] == 0
    assert np.all(e["idx"] == (1 << bits) // 2 - 1)
    assert np.all(e["sign_bits"] == 1)
    assert np.all(o.dequantize_rotated(e["idx"], e["norm16"], cent) == 0)


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_all_energy_on_channel_zero(bits, d):
    """x = a*s1: u = a*d*e_0 exactly, z_0 = sqrt(d) (top code), z_i = 0 otherwise."""
    cent, bnd = o.codebook(bits)
    s1 = o.rotation_signs(5, d)
    a = np.float32(0.5)
    x = (a * s1.astype(np.float32))[None, :]
    e = o.encode(x, s1, cent, bnd, bits)
    assert e["norm16"][0] == np.float16(0.5 * math.sqrt(d))
    L = 1 << bits
    assert e["idx"][0, 0] == L - 1
    assert np.all(e["idx"][0, 1:] == L // 2 - 1)


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("outliers", [False, True])
def test_distortion_matches_lloyd_max(bits, outliers):
    d, n = 128, 4000
    rng = np.random.default_rng(100 + bits)
    x = rng.standard_normal((n, d)).astype(np.float32)
    if outliers:
        x[:, [3, 17, 64, 100]] *= 20
    cent, bnd = o.codebook(bits)
    s1 = o.rotation_signs(9, d)
    e = o.encode(x, s1, cent, bnd, bits)
    xhat = o.rht_inverse(o.dequantize_rotated(e["idx"], e["norm16"], cent), s1)
    rel = np.sum((x - xhat) ** 2) / np.sum(x.astype(np.float64) ** 2)
    if not outliers:
        assert abs(rel - MAX_D[bits]) < 0.1 * MAX_D[bits]
        return
    # a few dominant channels: the rotated marginal is no longer Gaussian, but the
    # error stays at or below the Gaussian figure, far below quantizing unrotated
    assert rel < 1.1 * MAX_D[bits]
    nrm = np.linalg.norm(x.astype(np.float64), axis=1, keepdims=True)
    z = (math.sqrt(d) * x / nrm).astype(np.float32)
    plain = cent.astype(np.float64)[o.bucket_index(z, bnd)] * nrm / math.sqrt(d)
    rel_plain = np.sum((x - plain) ** 2) / np.sum(x.astype(np.float64) ** 2)
    assert rel < 0.5 * rel_plain


def test_norm_is_float32_then_fp16():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    e = o.encode(x, o.rotation_signs(0, 128), *o.codebook(3), 3)
    exact = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=1))
    np.testing.assert_allclose(e["norm16"].astype(np.float64), exact, rtol=2 ** -11)
    assert e["norm16"].dtype == np.float16


def test_qjl_residual_norm():
    d, bits = 128, 3
    rng = np.random.default_rng(6)
    x = rng.standard_normal((32, d)).astype(np.float32)
    cent, bnd = o.codebook(bits)
    s1, s2 = o.rotation_signs(1, d), o.rotation_signs(1, d, second=True)
    e = o.encode(x, s1, cent, bnd, bits, s2)
    resid = o.rht_forward(x, s1) - o.dequantize_rotated(e["idx"], e["norm16"], cent)
    np.testing.assert_allclose(e["rnorm16"].astype(np.float64), np.linalg.norm(resid, axis=1),
                               rtol=2e-3)
    # sign bits are the signs of R2 applied to the residual
    w = o.rht_forward(resid, s2)
    agree = (w >= 0) == (e["sign_bits"] == 1)
    assert agree.mean() > 0.995     # disagreements only where |w| is at float32 noise level
    assert np.all(agree | (np.abs(w) < 1e-4 * np.linalg.norm(resid, axis=1, keepdims=True)))


def _qjl_trial(seed, q, k, bits, cent, bnd):
    d = q.shape[0]
    s1, s2 = o.rotation_signs(seed, d), o.rotation_signs(seed, d, second=True)
    e = o.encode(k[None, :].astype(np.float32), s1, cent, bnd, bits, s2)
    q_rot = o.rht_forward(q, s1)
    khat = o.dequantize_rotated(e["idx"], e["norm16"], cent)[0]
    mse_only = float(q_rot @ khat)
    q_hat = o.rht_forward(q_rot, s2)
    sgn = 2.0 * e["sign_bits"][0] - 1.0
    rho = float(e["rnorm16"][0])
    corr = math.sqrt(math.pi / (2 * d)) * rho * float(q_hat @ sgn)
    r = o.rht_forward(k.astype(np.float64), s1) - khat
    return mse_only, corr, float(q_rot @ r), float(np.linalg.norm(r)), float(
        (q_rot @ r) / (np.linalg.norm(q_rot) * np.linalg.norm(r)))


@pytest.mark.parametrize("bits", [2, 3])
def test_qjl_unbiased_over_rotations(bits):
    d, n_seeds, cos = 128, 1500, 0.8
    rng = np.random.default_rng(77)
    k = rng.standard_normal(d)
    k /= np.linalg.norm(k)
    e = rng.standard_normal(d)
    e -= (e @ k) * k
    e /= np.linalg.norm(e)
    q = cos * k + math.sqrt(1 - cos * cos) * e
    cent, bnd = o.codebook(bits)
    trials = np.array([_qjl_trial(s, q, k.astype(np.float32).astype(np.float64), bits, cent, bnd)
                       for s in range(n_seeds)])
    true = float(q @ k.astype(np.float32).astype(np.float64))
    mse_err = trials[:, 0] - true
    qjl_err = trials[:, 0] + trials[:, 1] - true
    se = qjl_err.std(ddof=1) / math.sqrt(n_seeds)
    assert abs(qjl_err.mean()) < 3 * se
    # MSE-only scores are biased low by about cos * D_b (centroid condition E[y yhat] = E[yhat^2])
    assert mse_err.mean() < -8 * se
    assert abs(mse_err.mean() - (-cos * MAX_D[bits])) < 0.25 * cos * MAX_D[bits]
    # variance of the sketch around the true residual inner product
    noise = trials[:, 1] - trials[:, 2]
    pred = (math.pi / 2) * trials[:, 3] ** 2 / d * (1 - (2 / math.pi) * trials[:, 4] ** 2)
    # the Hadamard sketch's rows are exactly orthonormal, so its variance sits at or
    # below the i.i.d. Gaussian-sketch figure (about a third of it at d = 128)
    assert 0.1 * pred.mean() < noise.var() < 1.1 * pred.mean()
