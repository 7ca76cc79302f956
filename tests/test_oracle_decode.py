"""Pins of the oracle's decode attention (CPU only).

* two independent routes agree (rotated frame with the fast transform vs
  explicit rotation matrices and dequantized keys/values in the original frame);
* special cases: one token returns its dequantized value; identical keys return
  the mean of the dequantized values; one dominant score returns that value;
  an empty context returns zeros;
* the dense float64 reference equals torch's scaled_dot_product_attention;
* quality grows with the bit width (error vs unquantized attention 2 > 3 > 4 bits).
"""
import math

import numpy as np
import pytest
import torch

import oracle as o


def _cache(x_k, x_v, kb, vb, qjl, seed=0):
    d = x_k.shape[1]
    s1 = o.rotation_signs(seed, d)
    s2 = o.rotation_signs(seed, d, second=True) if qjl else None
    ck, bk = o.codebook(kb)
    cv, bv = o.codebook(vb)
    ek = o.encode(x_k, s1, ck, bk, kb, s2)
    ev = o.encode(x_v, s1, cv, bv, vb)
    kw = dict(s2=s2, k_sign_bits=ek.get("sign_bits"), k_rnorm16=ek.get("rnorm16"))
    return s1, ek, ev, ck, cv, kw


@pytest.mark.parametrize("qjl", [False, True])
@pytest.mark.parametrize("bits", [(3, 4), (2, 2), (4, 4)])
def test_two_routes_agree(qjl, bits):
    d, t, g = 128, 300, 4
    rng = np.random.default_rng(3)
    xk = rng.standard_normal((t, d)).astype(np.float32)
    xv = rng.standard_normal((t, d)).astype(np.float32)
    q = rng.standard_normal((g, d))
    s1, ek, ev, ck, cv, kw = _cache(xk, xv, bits[0], bits[1], qjl)
    a = o.decode_attention(q, s1, ek["idx"], ek["norm16"], ck, ev["idx"], ev["norm16"], cv, **kw)
    b = o.decode_attention_dequant_route(q, s1, ek["idx"], ek["norm16"], ck, ev["idx"],
                                         ev["norm16"], cv, **kw)
    np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12 * np.abs(b).max())


def test_single_token_returns_its_value():
    d = 128
    rng = np.random.default_rng(8)
    xk = rng.standard_normal((1, d)).astype(np.float32)
    xv = rng.standard_normal((1, d)).astype(np.float32)
    s1, ek, ev, ck, cv, kw = _cache(xk, xv, 3, 4, True)
    out = o.decode_attention(rng.standard_normal((2, d)), s1, ek["idx"], ek["norm16"], ck,
                             ev["idx"], ev["norm16"], cv, **kw)
    vhat = o.rht_inverse(o.dequantize_rotated(ev["idx"], ev["norm16"], cv), s1)[0]
    np.testing.assert_allclose(out, np.stack([vhat, vhat]), atol=1e-12)
    # the value itself is close to the input (4-bit distortion)
    assert np.sum((vhat - xv[0]) ** 2) / np.sum(xv[0].astype(np.float64) ** 2) < 0.05


def test_identical_keys_average_values():
    d, t = 128, 37
    rng = np.random.default_rng(9)
    xk = np.repeat(rng.standard_normal((1, d)).astype(np.float32), t, axis=0)
    xv = rng.standard_normal((t, d)).astype(np.float32)
    s1, ek, ev, ck, cv, kw = _cache(xk, xv, 2, 3, True)
    out = o.decode_attention(rng.standard_normal((1, d)), s1, ek["idx"], ek["norm16"], ck,
                             ev["idx"], ev["norm16"], cv, **kw)
    vhat = o.rht_inverse(o.dequantize_rotated(ev["idx"], ev["norm16"], cv), s1)
    np.testing.assert_allclose(out[0], vhat.mean(0), atol=1e-12)


def test_dominant_key_selects_its_value():
    d, t = 128, 64
    rng = np.random.default_rng(10)
    xk = rng.standard_normal((t, d)).astype(np.float32)
    xv = rng.standard_normal((t, d)).astype(np.float32)
    s1, ek, ev, ck, cv, kw = _cache(xk, xv, 4, 4, False)
    khat = o.rht_inverse(o.dequantize_rotated(ek["idx"], ek["norm16"], ck), s1)
    q = 500.0 * khat[17] / np.linalg.norm(khat[17])
    out = o.decode_attention(q, s1, ek["idx"], ek["norm16"], ck, ev["idx"], ev["norm16"], cv)
    vhat = o.rht_inverse(o.dequantize_rotated(ev["idx"], ev["norm16"], cv), s1)
    np.testing.assert_allclose(out[0], vhat[17], atol=1e-9)


def test_empty_context_is_zero():
    d = 64
    s1 = o.rotation_signs(0, d)
    ck, _ = o.codebook(3)
    e = np.zeros((0, d), np.int64)
    out = o.decode_attention(np.ones((3, d)), s1, e, np.zeros(0, np.float16), ck, e,
                             np.zeros(0, np.float16), ck)
    assert out.shape == (3, d) and np.all(out == 0)


def test_scale_default_and_explicit():
    d, t = 128, 50
    rng = np.random.default_rng(12)
    xk = rng.standard_normal((t, d)).astype(np.float32)
    xv = rng.standard_normal((t, d)).astype(np.float32)
    s1, ek, ev, ck, cv, kw = _cache(xk, xv, 3, 4, False)
    q = rng.standard_normal((1, d))
    args = (s1, ek["idx"], ek["norm16"], ck, ev["idx"], ev["norm16"], cv)
    a = o.decode_attention(q, *args)
    b = o.decode_attention(q, *args, sm_scale=1 / math.sqrt(d))
    c = o.decode_attention(q * 2, *args, sm_scale=0.5 / math.sqrt(d))
    np.testing.assert_allclose(a, b, atol=1e-14)
    np.testing.assert_allclose(a, c, atol=1e-12)


def test_dense_reference_matches_torch_sdpa():
    rng = np.random.default_rng(13)
    q = rng.standard_normal((4, 64))
    k = rng.standard_normal((100, 64))
    v = rng.standard_normal((100, 64))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None])[0].numpy()
    np.testing.assert_allclose(o.dense_attention(q, k, v), ref, atol=1e-12)


def test_quality_improves_with_bits():
    d, t = 128, 2000
    rng = np.random.default_rng(14)
    xk = rng.standard_normal((t, d)).astype(np.float32)
    xv = rng.standard_normal((t, d)).astype(np.float32)
    q = rng.standard_normal((8, d))
    dense = o.dense_attention(q, xk, xv)
    errs = []
    for b in (2, 3, 4):
        s1, ek, ev, ck, cv, kw = _cache(xk, xv, b, b, False)
        out = o.decode_attention(q, s1, ek["idx"], ek["norm16"], ck, ev["idx"], ev["norm16"], cv)
        errs.append(np.abs(out - dense).max())
    assert errs[0] > errs[1] > errs[2]


def test_kv_bits_split():
    assert o.kv_bits_split(3.5) == (3, 4)
    assert o.kv_bits_split(2.5) == (2, 3)
    assert o.kv_bits_split(4.0) == (4, 4)
    assert o.kv_bits_split(2) == (2, 2)
