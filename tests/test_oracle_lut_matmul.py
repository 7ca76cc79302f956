"""Pins of the oracle's weights-regime LUT matmul (blocks of d input channels
encoded as KV vectors, Y = X W_hat^T).

Tied to things outside the oracle's dequantization: the unquantized product
X W^T (numpy's matmul on the original W) must sit within the codec's
distortion; a second route that rotates the inputs and never forms W_hat must
agree; with one block the matmul must equal scores against the decode
oracle's dequantized keys.
"""
import math

import numpy as np
import pytest

import oracle as o

DISTORTION = {2: 0.1175, 3: 0.03455, 4: 0.009497}   # Max (1960), N(0,1)


def _weights(n, k, seed, outliers=True):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((n, k)).astype(np.float32)
    if outliers:
        w[:, rng.choice(k, 8, replace=False)] *= 20.0
    return w


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("outliers", [False, True])
def test_product_error_matches_the_codec_distortion(bits, d, outliers):
    n, k, m = 96, 4 * d, 6
    w = _weights(n, k, bits + d, outliers)
    cent, bnd = o.codebook(bits)
    s1 = o.rotation_signs(7, d)
    enc = o.weights_encode(w, s1, cent, bnd, bits)
    w_hat = o.weights_dequantize(enc["idx"], enc["norm16"], s1, cent)
    rel_w = np.sum((w_hat - w) ** 2) / np.sum(w.astype(np.float64) ** 2)
    if outliers:   # a few dominant channels: the rotated marginal is no longer Gaussian
        assert rel_w < 1.1 * DISTORTION[bits]
        return
    assert 0.85 * DISTORTION[bits] < rel_w < 1.15 * DISTORTION[bits]
    x = np.random.default_rng(1).standard_normal((m, k))
    y = o.lut_matmul(x, enc["idx"], enc["norm16"], s1, cent)
    exact = x @ w.astype(np.float64).T
    rel_y = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    assert 0.5 * math.sqrt(DISTORTION[bits]) < rel_y < 1.5 * math.sqrt(DISTORTION[bits])


def test_rotated_input_route_agrees():
    d, n, k = 128, 40, 512
    w = _weights(n, k, 3)
    cent, bnd = o.codebook(3)
    s1 = o.rotation_signs(11, d)
    enc = o.weights_encode(w, s1, cent, bnd, 3)
    x = np.random.default_rng(2).standard_normal((3, k))
    y = o.lut_matmul(x, enc["idx"], enc["norm16"], s1, cent)
    # sum over blocks of (n16 / sqrt(d)) <c[idx], R x_block>, W_hat never formed
    y2 = np.zeros_like(y)
    for j in range(k // d):
        xr = o.rht_forward(x[:, j * d:(j + 1) * d], s1)                      # [M][d]
        c = cent.astype(np.float64)[enc["idx"][j]]                          # [N][d]
        y2 += (xr @ c.T) * enc["norm16"][j].astype(np.float64)[None, :] / math.sqrt(d)
    assert np.allclose(y, y2, rtol=1e-11, atol=1e-9)


def test_single_block_equals_scores_on_dequantized_keys():
    d, n = 128, 50
    w = _weights(n, d, 5)
    cent, bnd = o.codebook(4)
    s1 = o.rotation_signs(0, d)
    enc = o.weights_encode(w, s1, cent, bnd, 4)
    e = o.encode(w, s1, cent, bnd, 4)                 # the same rows as KV keys
    keys = o.rht_inverse(o.dequantize_rotated(e["idx"], e["norm16"], cent), s1)
    x = np.random.default_rng(9).standard_normal((2, d))
    assert np.array_equal(enc["idx"][0], e["idx"])
    assert np.allclose(o.lut_matmul(x, enc["idx"], enc["norm16"], s1, cent), x @ keys.T,
                       rtol=1e-12, atol=1e-10)
