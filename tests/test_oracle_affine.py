"""Pins of the oracle's affine group-64 comparison codec (CPU only).

Cited: "mlx-turboquant" README, sections "Quantize the KV cache (long-context
inference)" (kv_group_size 64), "How it plugs in" (affine cache with rotated
keys; the attention rotates the query), "Measured results" (rotation rescues
low-bit affine KV) and "Memory footprint over long context" (bytes per token).

What pins it, other than itself:
* the pages' KB/token table (golden) against the per-vector byte count;
* vectors built on an affine grid with exact fp16 scale and bias come back bit
  for bit (codes, scale, bias, reconstruction);
* keys built as R^T y from a grid vector y, with R formed from the explicit
  Sylvester matrix: the codec returns y exactly and its decode equals textbook
  softmax attention on the unrotated keys;
* the rounding bound |y - y_hat| <= scale/2 plus the fp16 rounding of scale
  and bias, with min, max and range recomputed in float64;
* the rotated frame y against R x formed with the explicit matrix;
* the QJL residual norm and sign bits against an explicit-matrix second route.
"""
import math

import numpy as np
import pytest

import oracle as o


def _explicit_r(d, signs):
    return o.hadamard_matrix(d) * np.asarray(signs, np.float64)[None, :] / math.sqrt(d)


def _grid(rng, n, d, bits):
    """Codes (each group hits 0 and 2^b - 1), dyadic fp16-exact scales and
    nonzero biases, and the grid vectors b + s * c (exact in float32)."""
    lv = (1 << bits) - 1
    ng = d // 64
    c = rng.integers(0, lv + 1, (n, ng, 64))
    c[..., 0], c[..., 1] = 0, lv
    for i in range(n):                      # move the extremes off channel 0/1
        for g in range(ng):
            rng.shuffle(c[i, g])
    s = (1.0 + rng.integers(0, 8, (n, ng)) / 8.0) * 2.0 ** -rng.integers(2, 7, (n, ng)).astype(float)
    j = rng.integers(1, 64, (n, ng)) * rng.choice([-1, 1], (n, ng))
    b = j / 16.0
    y = (b[..., None] + s[..., None] * c).reshape(n, d)
    return c.reshape(n, d), s, b, y


def test_memory_footprint_table(golden):
    """The pages' KB/token table, from the byte layout: the fp16 row gives the
    cached channels per token and side; head_dim 128 (the only width that also
    fits the sketch row's per-vector norm)."""
    rows = {r[0]: (int(r[1]), int(r[2]), int(r[3]), float(r[4])) for r in golden("kv_memory_footprint.txt")}
    fp16 = rows.pop("fp16")
    channels = fp16[3] * 1024 / (2 * 2)        # per side (K or V), 2 bytes each
    d = 128
    vectors = channels / d
    for name, (kb, vb, qjl, kb_tok) in rows.items():
        per_token = (o.affine_vector_bytes(d, kb, bool(qjl)) + o.affine_vector_bytes(d, vb)) * vectors
        assert abs(per_token / 1024 - kb_tok) <= 0.05, name


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_values_on_grid_come_back_exactly(d, bits):
    rng = np.random.default_rng(10 * d + bits)
    c, s, b, y = _grid(rng, 9, d, bits)
    e = o.affine_encode(y.astype(np.float32), bits)
    assert np.array_equal(e["idx"], c)
    assert np.array_equal(e["scale16"].astype(np.float64), s)
    assert np.array_equal(e["bias16"].astype(np.float64), b)
    assert np.array_equal(o.affine_dequantize(e["idx"], e["scale16"], e["bias16"]), y)
    assert np.array_equal(o.unpack_codes(e["codes"], bits, d), c)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 4])
def test_rotated_keys_on_grid_and_decode_is_dense_attention(d, bits):
    rng = np.random.default_rng(7 * d + bits)
    s1 = o.rotation_signs(99, d)
    r = _explicit_r(d, s1)
    ck, _, _, yk = _grid(rng, 40, d, bits)
    cv, _, _, vals = _grid(rng, 40, d, bits)
    keys = yk @ r                              # rows R^T y
    ek = o.affine_encode(keys.astype(np.float32), bits, s1)
    assert np.array_equal(ek["idx"], ck)
    assert np.array_equal(o.affine_dequantize(ek["idx"], ek["scale16"], ek["bias16"]), yk)
    ev = o.affine_encode(vals.astype(np.float32), bits)
    assert np.array_equal(ev["idx"], cv)
    q = rng.standard_normal((4, d))
    got = o.affine_decode_attention(q, s1, ek, ev)
    want = o.dense_attention(q, keys, vals)
    assert np.allclose(got, want, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("rotate", [False, True])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_rounding_bound(rotate, bits):
    d = 128
    rng = np.random.default_rng(bits + 10 * rotate)
    x = rng.standard_normal((64, d)).astype(np.float32)
    x[:, [3, 70]] *= 25.0                                    # outlier channels
    s1 = o.rotation_signs(5, d) if rotate else None
    e = o.affine_encode(x, bits, s1)
    y = x.astype(np.float64) @ _explicit_r(d, s1).T if rotate else x.astype(np.float64)
    assert np.allclose(e["y"], y, rtol=0, atol=2e-5 * np.abs(y).max())   # the rotated frame
    lv = (1 << bits) - 1
    yg = e["y"].astype(np.float64).reshape(64, 2, 64)
    mn, mx = yg.min(-1), yg.max(-1)
    s = (mx - mn) / lv
    s16 = e["scale16"].astype(np.float64)
    b16 = e["bias16"].astype(np.float64)
    bound = s16 / 2 + np.abs(mn - b16) + lv * np.abs(s - s16) + 1e-6 * np.abs(yg).max(-1)
    err = np.abs(yg - o.affine_dequantize(e["idx"], e["scale16"], e["bias16"]).reshape(64, 2, 64)).max(-1)
    assert np.all(err <= bound)
    assert np.all(np.abs(s - s16) <= s * 2.0 ** -11 + 1e-12)
    assert np.all(np.abs(mn - b16) <= np.abs(mn) * 2.0 ** -11 + 2.0 ** -25)


def test_constant_group_has_zero_scale():
    x = np.ones((3, 128), np.float32) * np.float32(0.3)
    x[:, 64:] = np.linspace(-1, 1, 64, dtype=np.float32)
    e = o.affine_encode(x, 3)
    assert np.all(e["scale16"][:, 0] == 0) and np.all(e["idx"][:, :64] == 0)
    assert np.all(e["bias16"][:, 0] == np.float16(0.3))
    assert np.all(o.affine_dequantize(e["idx"], e["scale16"], e["bias16"])[:, :64] == float(np.float16(0.3)))


def test_groups_are_64_consecutive_channels():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((8, 256)).astype(np.float32)
    e0 = o.affine_encode(x, 4)
    x2 = x.copy()
    x2[:, 64:128] *= 7.0
    e1 = o.affine_encode(x2, 4)
    keep = np.r_[0:64, 128:256]
    assert np.array_equal(e0["idx"][:, keep], e1["idx"][:, keep])
    assert np.array_equal(e0["meta16"][:, [0, 1, 4, 5, 6, 7]], e1["meta16"][:, [0, 1, 4, 5, 6, 7]])
    assert not np.array_equal(e0["meta16"][:, 2:4], e1["meta16"][:, 2:4])


@pytest.mark.parametrize("d", [64, 128])
def test_qjl_sketch_second_route(d):
    rng = np.random.default_rng(d)
    s1, s2 = o.rotation_signs(11, d), o.rotation_signs(11, d, second=True)
    x = rng.standard_normal((32, d)).astype(np.float32)
    e = o.affine_encode(x, 3, s1, s2)
    y = x.astype(np.float64) @ _explicit_r(d, s1).T
    res = y - o.affine_dequantize(e["idx"], e["scale16"], e["bias16"])
    rho = np.linalg.norm(res, axis=1)
    assert np.allclose(e["rnorm16"].astype(np.float64), rho, rtol=2e-3)
    w = res @ _explicit_r(d, s2).T
    clear = np.abs(w) > 1e-4 * np.abs(w).max(axis=1, keepdims=True)
    assert np.array_equal(e["sign_bits"][clear], (w >= 0)[clear].astype(np.int64))


def test_decode_with_sketch_second_route():
    d = 128
    rng = np.random.default_rng(21)
    s1, s2 = o.rotation_signs(4, d), o.rotation_signs(4, d, second=True)
    k = rng.standard_normal((50, d)).astype(np.float32)
    v = rng.standard_normal((50, d)).astype(np.float32)
    ek = o.affine_encode(k, 3, s1, s2)
    ev = o.affine_encode(v, 3)
    q = rng.standard_normal((2, d))
    got = o.affine_decode_attention(q, s1, ek, ev, s2=s2)
    r1, r2 = _explicit_r(d, s1), _explicit_r(d, s2)
    keys = o.affine_dequantize(ek["idx"], ek["scale16"], ek["bias16"]) @ r1      # R^T k_hat
    sgn = 2.0 * ek["sign_bits"] - 1.0
    sc = q @ keys.T + math.sqrt(math.pi / (2 * d)) * ek["rnorm16"].astype(np.float64)[None] * ((q @ r1.T @ r2.T) @ sgn.T)
    sc /= math.sqrt(d)
    p = np.exp(sc - sc.max(1, keepdims=True))
    want = p @ o.affine_dequantize(ev["idx"], ev["scale16"], ev["bias16"]) / p.sum(1, keepdims=True)
    assert np.allclose(got, want, rtol=1e-9, atol=1e-12)


def test_empty_cache_gives_zero():
    d = 64
    e = o.affine_encode(np.zeros((0, d), np.float32), 2, o.rotation_signs(0, d))
    assert o.affine_decode_attention(np.ones((3, d)), o.rotation_signs(0, d), e, e).shape == (3, d)
    assert not o.affine_decode_attention(np.ones((3, d)), o.rotation_signs(0, d), e, e).any()


def test_rotation_rescues_outlier_keys():
    """The pages' measured effect, on synthetic keys with a few large channels:
    at 4 bits the rotated affine code scores the keys more accurately than the
    plain one (the rotation spreads an outlier over every channel)."""
    d, t = 128, 512
    rng = np.random.default_rng(8)
    k = rng.standard_normal((t, d)).astype(np.float32)
    k[:, [5, 17, 90, 101]] *= 20.0
    q = rng.standard_normal((16, d))
    s1 = o.rotation_signs(2, d)
    exact = q @ k.T.astype(np.float64)
    plain = o.affine_encode(k, 4)
    rot = o.affine_encode(k, 4, s1)
    err_plain = q @ o.affine_dequantize(plain["idx"], plain["scale16"], plain["bias16"]).T - exact
    err_rot = o.rht_forward(q, s1) @ o.affine_dequantize(rot["idx"], rot["scale16"], rot["bias16"]).T - exact
    assert np.sqrt((err_rot ** 2).mean()) < 0.7 * np.sqrt((err_plain ** 2).mean())


def test_zero_extremes_are_positive_zero():
    """-0 and +0 are one value: a group whose min or max is a zero stores it as +0."""
    x = np.zeros((3, 128), np.float32)
    x[1] = -0.0                                                       # all -0
    x[2, :64] = np.where(np.arange(64) % 2, -0.0, 0.0)                # mixed zeros
    x[2, 64:] = -np.linspace(-1, 0, 64, dtype=np.float32)             # 1 .. -0: min is -0
    for s1 in (None, o.rotation_signs(1, 128)):
        assert not np.any(o.affine_encode(x, 3, s1)["meta16"][:2].view(np.uint16) & 0x8000)
    assert o.affine_encode(x, 3)["meta16"][2].view(np.uint16).tolist()[:2] == [0, 0]
    assert o.affine_encode(x, 3)["meta16"][2].view(np.uint16)[3] == 0     # bias of group 1: +0
