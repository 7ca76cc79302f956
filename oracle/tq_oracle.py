"""Plain CPU oracle for the TurboQuant KV-cache codec and fused decode attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline legs of ``bench.py``, never by the product path.  It shares no
code, table or constant generator with the CUDA library; it imports numpy, the
Python standard library and, for the unit-sphere codebook only, scipy.special.

Sources, cited by page title and section:

* [P1] "TurboQuant Performance Benefits: Memory Reduction and Speed Optimization
  in MLX-VLM" -- "What Is TurboQuant?" (random Hadamard rotation, then MSE
  codebook quantization at 2-4 bits per dimension), "Fractional-Bit Precision
  Support" (3.5 bits = 3-bit keys + 4-bit values), "Custom Metal Kernel
  Implementation" (scores and value aggregation computed on packed codes).
* [P2] "How to Use TurboQuant with the MLX-VLM Python API: A Complete Guide" --
  "What is TurboQuant?" (``_rotation_matrix``, ``_rht_forward``,
  ``_rht_inverse``, ``_codebook``; fused scoring on packed low-bit data).
* [P3] "mlx-turboquant" README -- introduction (randomized Hadamard transform
  preserves inner products, Lloyd-Max codebook), "The 1-bit QJL residual
  (unbiased inner-product estimator)" (r = Rk - k_hat, store sign(RHT2(r)) and
  ||r||, add sqrt(pi/(2d))*||r||*<RHT2(Rq), sign(RHT2(r))> back to the score);
  for the affine comparison codec: "Quantize the KV cache (long-context
  inference)" (kv_group_size 64), "How it plugs in" (affine cache, rotated keys,
  rotated query), "Measured results" and "Memory footprint over long context".

Precision.  The codec is computed in IEEE binary32 with round-to-nearest-even,
one operation at a time (numpy float32 ufuncs never fuse a multiply into an add),
in a fixed operation order: its integer outputs (codes, sign bits) and its fp16
norms are compared bit for bit.  The Lloyd-Max solve and the attention are
computed in binary64.

Readings taken where the pages are silent (each one is also listed in the design
notes): one Sylvester-ordered Hadamard round per rotation, R = H D1 / sqrt(d);
sign vectors from SplitMix64 (top bit of each output, channel 0 first; the second
rotation uses seed XOR 0x9E3779B97F4A7C15); one rotation shared by keys, values
and all heads; a Lloyd-Max codebook for N(0, 1) applied to z = sqrt(d) * Rx /
||x||; a per-vector fp16 norm; codes packed as a little-endian bit stream;
strict "<" against the boundaries (a tie goes to the lower index); sign(0) = +1;
the QJL residual norm kept in the orthonormal rotated frame.  Affine codec:
groups of 64 consecutive channels, scale = (max - min)/(2^b - 1) and bias = min
in fp16, codes rounded half to even and clamped, keys coded in the rotated frame
and values unrotated.

Parity status: every function is pinned by the CPU tests in ``tests/`` against
closed forms, textbook tables, brute force or an independent second route; none
is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

MASK64 = (1 << 64) - 1
# SplitMix64's additive constant (Steele, Lea & Flood, "Fast splittable
# pseudorandom number generators", OOPSLA 2014); also used to derive the seed of
# the second rotation.
GOLDEN64 = 0x9E3779B97F4A7C15


# ---------------------------------------------------------------------------
# Random signs of the randomized Hadamard transform  ([P2] "What is
# TurboQuant?": _rotation_matrix; [P3] introduction: "Randomized Hadamard
# Transform").  The pages do not give the generator; SplitMix64 is used.
# ---------------------------------------------------------------------------
def splitmix64(seed: int, n: int) -> list[int]:
    """The first ``n`` outputs of SplitMix64 started from state ``seed``.

    Published definition: state += 0x9E3779B97F4A7C15; z = state;
    z = (z ^ z>>30) * 0xBF58476D1CE4E5B9; z = (z ^ z>>27) * 0x94D049BB133111EB;
    output z ^ z>>31, all modulo 2**64.
    """
    state = seed & MASK64
    out = []
    for _ in range(n):
        state = (state + GOLDEN64) & MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        out.append(z ^ (z >> 31))
    return out


def rotation_signs(seed: int, d: int, second: bool = False) -> np.ndarray:
    """Diagonal of D (entries +1/-1) for channel 0..d-1.

    Channel i takes the i-th SplitMix64 output and is -1 when its top bit is set.
    ``second=True`` gives D2 of the QJL rotation RHT2, seeded with
    seed XOR 0x9E3779B97F4A7C15.
    """
    state = (seed ^ GOLDEN64) if second else seed
    return np.array([-1 if (w >> 63) else 1 for w in splitmix64(state, d)],
                    dtype=np.int8)


def hadamard_matrix(d: int) -> np.ndarray:
    """Sylvester Hadamard matrix in natural order: H[i, j] = (-1)^popcount(i & j)."""
    i = np.arange(d, dtype=np.int64)
    parity = np.bitwise_count(i[:, None] & i[None, :]) & 1
    return np.where(parity == 0, 1.0, -1.0)


def fwht(v: np.ndarray, dtype=np.float32) -> np.ndarray:
    """Unnormalized Walsh-Hadamard transform u = H v along the last axis.

    Canonical butterfly order: for h = 1, 2, 4, ..., d/2 and every j whose bit h
    is clear, (v[j], v[j+h]) <- (v[j] + v[j+h], v[j] - v[j+h]).  Each add and
    subtract is rounded to ``dtype`` on its own.
    """
    v = np.array(v, dtype=dtype, copy=True)
    d = v.shape[-1]
    assert d & (d - 1) == 0, "head_dim must be a power of two"
    lead = v.shape[:-1]
    h = 1
    while h < d:
        w = v.reshape(lead + (d // (2 * h), 2, h))
        a = w[..., 0, :].copy()
        b = w[..., 1, :].copy()
        w[..., 0, :] = a + b
        w[..., 1, :] = a - b
        v = w.reshape(lead + (d,))
        h *= 2
    return v


def rht_forward(x: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """R x with R = H D / sqrt(d), in float64 ([P2] _rht_forward)."""
    x = np.asarray(x, np.float64)
    return fwht(signs * x, np.float64) / math.sqrt(x.shape[-1])


def rht_inverse(y: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """R^T y = D H y / sqrt(d), in float64 ([P2] _rht_inverse)."""
    y = np.asarray(y, np.float64)
    return signs * fwht(y, np.float64) / math.sqrt(y.shape[-1])


def pairwise_sum_f32(x: np.ndarray) -> np.ndarray:
    """Balanced pairwise sum over the last axis in float32.

    Level 1 adds (0+1), (2+3), ...; every later level adds adjacent pairs of the
    previous level's partial sums.  The length must be a power of two.
    """
    x = np.asarray(x, np.float32)
    while x.shape[-1] > 1:
        x = x[..., 0::2] + x[..., 1::2]
    return x[..., 0]


# ---------------------------------------------------------------------------
# Lloyd-Max MSE codebook for N(0, 1)  ([P2] "What is TurboQuant?": _codebook;
# [P3] introduction: "Lloyd-Max"; the rotated coordinates are near-Gaussian).
# ---------------------------------------------------------------------------
_SQRT2 = math.sqrt(2.0)
_INV_SQRT_2PI = 1.0 / math.sqrt(2.0 * math.pi)


def _pdf(x: float) -> float:
    return 0.0 if math.isinf(x) else math.exp(-0.5 * x * x) * _INV_SQRT_2PI


def _upper_tail(x: float) -> float:
    """P(X > x) for X ~ N(0, 1)."""
    return 0.5 * math.erfc(x / _SQRT2)


def gaussian_mass(a: float, b: float) -> float:
    """P(a < X < b) for X ~ N(0, 1), written so that no tail cancels."""
    if a >= 0.0:
        return _upper_tail(a) - _upper_tail(b)
    if b <= 0.0:
        return _upper_tail(-b) - _upper_tail(-a)
    return 1.0 - _upper_tail(-a) - _upper_tail(b)


def gaussian_cell_mean(a: float, b: float) -> float:
    """E[X | a < X < b] = (pdf(a) - pdf(b)) / P(a < X < b)."""
    return (_pdf(a) - _pdf(b)) / gaussian_mass(a, b)


def lloyd_max_gaussian(levels: int, init=None, tol: float = 1e-14,
                       max_iter: int = 1_000_000) -> tuple[np.ndarray, int]:
    """Lloyd's iteration for the MSE-optimal ``levels``-point quantizer of N(0,1).

    Alternates the two optimality conditions until no centroid moves by more
    than ``tol``: every boundary is the midpoint of its two neighbouring
    centroids, and every centroid is the conditional mean of its cell.  Returns
    (centroids ascending, float64; iterations used).
    """
    if init is None:
        # spread the start points evenly over [-2, 2]
        c = [(-2.0 + 4.0 * (j + 0.5) / levels) for j in range(levels)]
    else:
        c = [float(t) for t in init]
    for it in range(1, max_iter + 1):
        edges = [-math.inf] + [(c[j] + c[j + 1]) / 2 for j in range(levels - 1)] + [math.inf]
        new = [gaussian_cell_mean(edges[j], edges[j + 1]) for j in range(levels)]
        moved = max(abs(n - o) for n, o in zip(new, c))
        c = new
        if moved < tol:
            return np.array(c, np.float64), it
    raise RuntimeError("Lloyd-Max iteration did not converge")


def codebook(bits: int) -> tuple[np.ndarray, np.ndarray]:
    """(centroids, boundaries) in float32 for a ``bits``-bit code.

    The float64 Lloyd-Max solution is made exactly odd-symmetric (each positive
    centroid averaged with its negated mirror), rounded to float32, and the
    negative half is the negation of the positive half.  Boundary j is
    (c[j] + c[j+1]) * 0.5 evaluated in float32, so the middle one is exactly 0.
    """
    levels = 1 << bits
    c64, _ = lloyd_max_gaussian(levels)
    half = levels // 2
    pos = np.array([(c64[half + j] - c64[half - 1 - j]) / 2 for j in range(half)],
                   dtype=np.float32)
    cent = np.concatenate([-pos[::-1], pos]).astype(np.float32)
    bnd = ((cent[:-1] + cent[1:]) * np.float32(0.5)).astype(np.float32)
    return cent, bnd


# ---------------------------------------------------------------------------
# Codebook for the exact distribution of a rotated coordinate.  [P3]'s
# introduction calls the rotated coordinates near-Gaussian, which is what the
# N(0,1) codebook above assumes.  Exactly: for a fixed vector x, each
# coordinate of R x / ||x|| is a coordinate of a uniformly random unit vector
# of R^d, so z = sqrt(d) * (R x)_i / ||x|| has density
#     f_d(z) = C_d * (1 - z^2/d)^((d-3)/2)  on |z| < sqrt(d),
#     C_d = Gamma(d/2) / (sqrt(pi d) Gamma((d-1)/2)),
# and z^2/d ~ Beta(1/2, (d-1)/2).  f_d tends to the N(0,1) density as d grows.

def sphere_density(z: float, d: int) -> float:
    if abs(z) >= math.sqrt(d):
        return 0.0
    c = math.exp(math.lgamma(d / 2) - math.lgamma((d - 1) / 2)) / math.sqrt(math.pi * d)
    return c * (1.0 - z * z / d) ** ((d - 3) / 2)


def _sphere_upper_tail(z: float, d: int) -> float:
    """P(Z > z) for z >= 0: half of P(Z^2/d > z^2/d) (the complemented
    regularized incomplete beta function, so no tail cancels)."""
    from scipy.special import betaincc
    if z >= math.sqrt(d):
        return 0.0
    return 0.5 * float(betaincc(0.5, (d - 1) / 2, z * z / d))


def sphere_mass(a: float, b: float, d: int) -> float:
    """P(a < Z < b) for the scaled coordinate Z of a random unit vector of R^d."""
    if a >= 0.0:
        return _sphere_upper_tail(a, d) - _sphere_upper_tail(b, d)
    if b <= 0.0:
        return _sphere_upper_tail(-b, d) - _sphere_upper_tail(-a, d)
    return 1.0 - _sphere_upper_tail(-a, d) - _sphere_upper_tail(b, d)


def sphere_first_moment(a: float, b: float, d: int) -> float:
    """Integral of z f_d(z) over (a, b): an antiderivative of z (1 - z^2/d)^k is
    -(d / (2 (k + 1))) (1 - z^2/d)^(k + 1), here with k = (d - 3)/2."""
    r = math.sqrt(d)
    a, b = max(a, -r), min(b, r)
    c = math.exp(math.lgamma(d / 2) - math.lgamma((d - 1) / 2)) / math.sqrt(math.pi * d)
    g = lambda z: max(0.0, 1.0 - z * z / d) ** ((d - 1) / 2)
    return c * d / (d - 1) * (g(a) - g(b))


def sphere_cell_mean(a: float, b: float, d: int) -> float:
    """E[Z | a < Z < b]."""
    return sphere_first_moment(a, b, d) / sphere_mass(a, b, d)


def lloyd_max_sphere(levels: int, d: int, init=None, tol: float = 1e-14,
                     max_iter: int = 1_000_000) -> tuple[np.ndarray, int]:
    """Lloyd's iteration (midpoint boundaries, conditional-mean centroids) for
    the density f_d; starts from the N(0,1) solution unless ``init`` is given."""
    c = [float(t) for t in (lloyd_max_gaussian(levels)[0] if init is None else init)]
    for it in range(1, max_iter + 1):
        edges = [-math.inf] + [(c[j] + c[j + 1]) / 2 for j in range(levels - 1)] + [math.inf]
        new = [sphere_cell_mean(edges[j], edges[j + 1], d) for j in range(levels)]
        moved = max(abs(n - o) for n, o in zip(new, c))
        c = new
        if moved < tol:
            return np.array(c, np.float64), it
    raise RuntimeError("Lloyd-Max iteration did not converge")


def sphere_codebook(bits: int, d: int) -> tuple[np.ndarray, np.ndarray]:
    """(centroids, boundaries) in float32 for the density f_d, made odd-symmetric
    and rounded exactly as ``codebook`` does for N(0,1)."""
    levels = 1 << bits
    c64, _ = lloyd_max_sphere(levels, d)
    half = levels // 2
    pos = np.array([(c64[half + j] - c64[half - 1 - j]) / 2 for j in range(half)],
                   dtype=np.float32)
    cent = np.concatenate([-pos[::-1], pos]).astype(np.float32)
    bnd = ((cent[:-1] + cent[1:]) * np.float32(0.5)).astype(np.float32)
    return cent, bnd


def bucket_index(z: np.ndarray, boundaries: np.ndarray) -> np.ndarray:
    """Code of each coordinate: the number of boundaries strictly below it."""
    idx = np.zeros(np.shape(z), np.int64)
    for b in boundaries:
        idx += (b < z)
    return idx


# ---------------------------------------------------------------------------
# Packed storage ([P1] "Custom Metal Kernel Implementation": kernels read packed
# data; [P3] "Roadmap": 3-bit packing).  Layout: per vector, a little-endian bit
# stream in which channel i's b-bit code occupies bits [b*i, b*i + b), bit 0
# being the least significant bit of byte 0.
# ---------------------------------------------------------------------------
def pack_codes(idx: np.ndarray, bits: int) -> np.ndarray:
    idx = np.asarray(idx, np.int64)
    n, d = idx.shape
    bitarr = ((idx[..., None] >> np.arange(bits)) & 1).astype(np.uint8)
    return np.packbits(bitarr.reshape(n, d * bits), axis=-1, bitorder="little")


def unpack_codes(packed: np.ndarray, bits: int, d: int) -> np.ndarray:
    packed = np.asarray(packed, np.uint8)
    n = packed.shape[0]
    stream = np.unpackbits(packed, axis=-1, bitorder="little")[:, :d * bits]
    bitarr = stream.reshape(n, d, bits).astype(np.int64)
    return (bitarr << np.arange(bits)).sum(-1)


# ---------------------------------------------------------------------------
# Codec (one vector per row)
# ---------------------------------------------------------------------------
def encode(x: np.ndarray, s1: np.ndarray, centroids: np.ndarray,
           boundaries: np.ndarray, bits: int, s2: np.ndarray | None = None) -> dict:
    """Quantize the rows of ``x`` (float32 [N, d]).

    Steps, each rounded to float32:
      1. n = sqrt(pairwise sum of x_i*x_i); n16 = fp16(n)            (per-vector norm)
      2. u = H (s1 * x)                     (sign flips, then unnormalized WHT)
      3. z = u * (1/n), with 1/n := 0 when n == 0  (= sqrt(d) * Rx / ||x||)
      4. idx_i = #{j : boundary_j < z_i}           (Lloyd-Max codebook)
      5. codes = little-endian bit stream of idx
    With ``s2`` given (QJL residual sketch of [P3] "The 1-bit QJL residual"):
      6. r = u - n16 * c[idx]            (residual, sqrt(d) times Rk - k_hat)
      7. rho = sqrt(pairwise sum of r_i*r_i) / sqrt(d); rho16 = fp16(rho)  (= ||Rk - k_hat||)
      8. w = H (s2 * r); sign bit_i = (w_i >= 0), so sign(0) = +1
    """
    x = np.asarray(x, np.float32)
    d = x.shape[-1]
    n = np.sqrt(pairwise_sum_f32(x * x))
    n16 = n.astype(np.float16)
    u = fwht(np.where(s1 < 0, -x, x))
    inv = np.zeros_like(n)
    nz = n != 0
    inv[nz] = np.float32(1.0) / n[nz]
    z = u * inv[:, None]
    idx = bucket_index(z, boundaries)
    out = {"idx": idx, "codes": pack_codes(idx, bits), "norm16": n16}
    if s2 is not None:
        r = u - n16.astype(np.float32)[:, None] * centroids[idx]
        rho = np.sqrt(pairwise_sum_f32(r * r)) / np.sqrt(np.float32(d))
        w = fwht(np.where(s2 < 0, -r, r))
        sbits = (w >= 0).astype(np.int64)
        out.update(sign_bits=sbits, signs=pack_codes(sbits, 1),
                   rnorm16=rho.astype(np.float16))
    return out


def dequantize_rotated(idx: np.ndarray, norm16: np.ndarray, centroids: np.ndarray) -> np.ndarray:
    """Reconstruction in the orthonormal rotated frame: n16 * c[idx] / sqrt(d) (float64)."""
    d = idx.shape[-1]
    return (np.asarray(norm16, np.float64)[:, None]
            * np.asarray(centroids, np.float64)[idx] / math.sqrt(d))


# ---------------------------------------------------------------------------
# Decode attention on the compressed cache ([P1] "Custom Metal Kernel
# Implementation": score and aggregate on packed codes; [P3] "The 1-bit QJL
# residual": the correction term; [P2] _rht_inverse for the output).
# ---------------------------------------------------------------------------
def default_scale(d: int, sm_scale: float | None) -> float:
    return 1.0 / math.sqrt(d) if (sm_scale is None or sm_scale <= 0) else float(sm_scale)


def decode_attention(q: np.ndarray, s1: np.ndarray, k_idx: np.ndarray, k_norm16: np.ndarray,
                     ck: np.ndarray, v_idx: np.ndarray, v_norm16: np.ndarray, cv: np.ndarray,
                     sm_scale: float | None = None, s2: np.ndarray | None = None,
                     k_sign_bits: np.ndarray | None = None,
                     k_rnorm16: np.ndarray | None = None) -> np.ndarray:
    """Attention of the G query rows ``q`` [G, d] over T cached tokens of one KV head.

    Rotated-frame route, float64:
      q_rot = R q;  k_hat_t = n16_t c_K[idx_t] / sqrt(d);  v_hat_t likewise
      s_t = scale * (<q_rot, k_hat_t> + sqrt(pi/(2d)) * rho16_t * <R2 q_rot, 2 b_t - 1>)
            (the second term only with the QJL sketch)
      p = softmax(s);  o = R^T (sum_t p_t v_hat_t)
    T = 0 gives a zero output.
    """
    q = np.atleast_2d(np.asarray(q, np.float64))
    g, d = q.shape
    t = k_idx.shape[0]
    if t == 0:
        return np.zeros((g, d))
    scale = default_scale(d, sm_scale)
    q_rot = rht_forward(q, s1)
    scores = q_rot @ dequantize_rotated(k_idx, k_norm16, ck).T
    if s2 is not None:
        q_hat = rht_forward(q_rot, s2)
        sgn = 2.0 * np.asarray(k_sign_bits, np.float64) - 1.0
        scores = scores + (math.sqrt(math.pi / (2 * d))
                           * np.asarray(k_rnorm16, np.float64)[None, :] * (q_hat @ sgn.T))
    scores = scale * scores
    p = np.exp(scores - scores.max(axis=-1, keepdims=True))
    o_rot = (p @ dequantize_rotated(v_idx, v_norm16, cv)) / p.sum(axis=-1, keepdims=True)
    return rht_inverse(o_rot, s1)


def decode_attention_dequant_route(q, s1, k_idx, k_norm16, ck, v_idx, v_norm16, cv,
                                   sm_scale=None, s2=None, k_sign_bits=None, k_rnorm16=None):
    """Second route for cross-checking ``decode_attention``.

    Builds R = H D1 / sqrt(d) and R2 = H D2 / sqrt(d) as explicit matrices from
    ``hadamard_matrix``, dequantizes every key and value back to the original
    frame (R^T k_hat), and runs dense softmax attention against the unrotated
    query; the QJL estimate is formed as sqrt(pi/(2d)) * rho * <R2 R q, 2b - 1>.
    """
    q = np.atleast_2d(np.asarray(q, np.float64))
    g, d = q.shape
    if k_idx.shape[0] == 0:
        return np.zeros((g, d))
    hm = hadamard_matrix(d)
    r1 = hm * np.asarray(s1, np.float64)[None, :] / math.sqrt(d)
    keys = dequantize_rotated(k_idx, k_norm16, ck) @ r1          # rows: R^T k_hat
    vals = dequantize_rotated(v_idx, v_norm16, cv) @ r1
    scores = q @ keys.T
    if s2 is not None:
        r2 = hm * np.asarray(s2, np.float64)[None, :] / math.sqrt(d)
        sgn = 2.0 * np.asarray(k_sign_bits, np.float64) - 1.0
        scores = scores + (math.sqrt(math.pi / (2 * d)) * np.asarray(k_rnorm16, np.float64)[None, :]
                           * ((q @ r1.T @ r2.T) @ sgn.T))
    scores = default_scale(d, sm_scale) * scores
    p = np.exp(scores - scores.max(axis=-1, keepdims=True))
    return (p @ vals) / p.sum(axis=-1, keepdims=True)


def dense_attention(q: np.ndarray, keys: np.ndarray, vals: np.ndarray,
                    sm_scale: float | None = None) -> np.ndarray:
    """Unquantized softmax attention in float64: q [G, d], keys/vals [T, d]."""
    q = np.atleast_2d(np.asarray(q, np.float64))
    keys = np.asarray(keys, np.float64)
    vals = np.asarray(vals, np.float64)
    if keys.shape[0] == 0:
        return np.zeros(q.shape)
    s = default_scale(q.shape[-1], sm_scale) * (q @ keys.T)
    p = np.exp(s - s.max(axis=-1, keepdims=True))
    return (p @ vals) / p.sum(axis=-1, keepdims=True)


# ---------------------------------------------------------------------------
# Weights regime ([P3] introduction: "Weights (MSE regime)": rotate each weight
# matrix, then quantize; "The Metal kernels" item 1: a non-uniform LUT dequant
# + matmul computed directly on packed indices).  Reading: each row of
# W [N][K] is cut into K/d blocks of d input channels, and every block is
# encoded exactly as a KV vector is (fp16 norm, rotation, Lloyd-Max codes).
# ---------------------------------------------------------------------------
def weights_encode(w: np.ndarray, s1: np.ndarray, centroids: np.ndarray,
                   boundaries: np.ndarray, bits: int) -> dict:
    """w float32 [N][K] -> idx [K/d][N][d], codes [K/d][N][bits*d/8], norm16 [K/d][N]
    (block j of every row is encoded by ``encode``; d = len(s1))."""
    w = np.asarray(w, np.float32)
    d = len(s1)
    n, k = w.shape
    blocks = w.reshape(n, k // d, d).transpose(1, 0, 2)
    enc = [encode(blocks[j], s1, centroids, boundaries, bits) for j in range(k // d)]
    return {key: np.stack([e[key] for e in enc]) for key in ("idx", "codes", "norm16")}


def weights_dequantize(idx: np.ndarray, norm16: np.ndarray, s1: np.ndarray,
                       centroids: np.ndarray) -> np.ndarray:
    """W_hat float64 [N][K]: block j of row n is R^T (n16 c[idx] / sqrt(d))."""
    blocks = [rht_inverse(dequantize_rotated(idx[j], norm16[j], centroids), s1)
              for j in range(idx.shape[0])]
    return np.concatenate(blocks, axis=1)


def lut_matmul(x: np.ndarray, idx: np.ndarray, norm16: np.ndarray, s1: np.ndarray,
               centroids: np.ndarray) -> np.ndarray:
    """Y = X W_hat^T in float64 for X [M][K]."""
    return np.asarray(x, np.float64) @ weights_dequantize(idx, norm16, s1, centroids).T


def kv_bits_split(kv_bits: float) -> tuple[int, int]:
    """Key and value bit widths for a (possibly fractional) kv_bits.

    [P1] "Fractional-Bit Precision Support": 3.5 bits = 3-bit keys, 4-bit values,
    read as keys floor(b), values ceil(b).
    """
    return int(math.floor(kv_bits + 1e-9)), int(math.ceil(kv_bits - 1e-9))


# ---------------------------------------------------------------------------
# Rotated affine group-64 KV codec, the comparison codec ([P3] "Quantize the KV
# cache (long-context inference)": kv_bits with kv_group_size=64; "How it plugs
# in": the KV cache is mlx-lm's affine quantized cache with the keys rotated,
# and the attention rotates the query and, with qjl, adds the sketch term;
# "Measured results": plain affine KV versus the rotated one; "Memory footprint
# over long context": the bytes per token).  Readings: a group is 64 consecutive
# channels of a vector; per group, scale = (max - min) / (2^b - 1) and
# bias = min, both stored as fp16, and a channel's code is
# round((y - bias) / scale) clamped to [0, 2^b - 1]; keys are coded in the
# rotated frame y = R k, values in their own frame (no rotation), so the
# attention output needs no inverse rotation; the QJL sketch codes the residual
# r = y - y_hat of the keys exactly as for the Lloyd-Max codec.
# ---------------------------------------------------------------------------
AFFINE_GROUP = 64


def affine_encode(x: np.ndarray, bits: int, s1: np.ndarray | None = None,
                  s2: np.ndarray | None = None) -> dict:
    """Affine group-64 coding of the rows of ``x`` (float32 [N, d]).

    Steps, each rounded to float32 (``s1`` None: no rotation, the plain codec):
      1. y = H (s1 * x) * rs, rs = fp32(1 / fp32(sqrt(d)))     (= R x, rounded)
      2. per group of 64 channels: mn = min y, mx = max y, each plus +0 (the
         extremes are values: -0 and +0 are equal, and a zero extreme is +0)
      3. scale16 = fp16((mx - mn) / (2^b - 1)); bias16 = fp16(mn)
      4. idx = rint((y - bias16) / scale16), ties to even, clamped to
         [0, 2^b - 1]; idx = 0 where scale16 == 0 (or the quotient is NaN)
      5. codes = little-endian bit stream of idx
    With ``s2`` (keys with the QJL sketch):
      6. y_hat = fp32(fp32(scale16 * idx) + bias16); r = y - y_hat
      7. rho = sqrt(pairwise sum of r_i * r_i); rnorm16 = fp16(rho)    (= ||Rk - k_hat||)
      8. w = H (s2 * r); sign bit_i = (w_i >= 0)
    ``meta16`` interleaves (scale16, bias16) per group: fp16 [N, 2 d / 64].
    """
    x = np.asarray(x, np.float32)
    n, d = x.shape
    ng = d // AFFINE_GROUP
    if s1 is not None:
        rs = np.float32(1.0) / np.sqrt(np.float32(d))
        y = fwht(np.where(s1 < 0, -x, x)) * rs
    else:
        y = x.copy()
    yg = y.reshape(n, ng, AFFINE_GROUP)
    mn = yg.min(axis=-1) + np.float32(0.0)       # as values: a zero extreme is +0
    mx = yg.max(axis=-1) + np.float32(0.0)
    levels = np.float32((1 << bits) - 1)
    scale16 = ((mx - mn) / levels).astype(np.float16)
    bias16 = mn.astype(np.float16)
    sf = scale16.astype(np.float32)[..., None]
    bf = bias16.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.rint((yg - bf) / sf)
    t = np.where(np.isnan(t) | (sf == 0), np.float32(0), t)
    idx = np.clip(t, 0, levels).astype(np.int64).reshape(n, d)
    meta = np.stack([scale16, bias16], axis=-1).reshape(n, 2 * ng)
    out = {"idx": idx, "codes": pack_codes(idx, bits), "scale16": scale16, "bias16": bias16,
           "meta16": meta, "y": y}
    if s2 is not None:
        y_hat = (sf * idx.reshape(n, ng, AFFINE_GROUP).astype(np.float32) + bf).reshape(n, d)
        r = y - y_hat
        rho = np.sqrt(pairwise_sum_f32(r * r))
        w = fwht(np.where(s2 < 0, -r, r))
        sbits = (w >= 0).astype(np.int64)
        out.update(sign_bits=sbits, signs=pack_codes(sbits, 1), rnorm16=rho.astype(np.float16))
    return out


def affine_dequantize(idx: np.ndarray, scale16: np.ndarray, bias16: np.ndarray) -> np.ndarray:
    """y_hat = scale16 * idx + bias16 per group, in float64 ([N, d])."""
    idx = np.asarray(idx, np.float64)
    n, d = idx.shape
    ng = d // AFFINE_GROUP
    s = np.asarray(scale16, np.float64).reshape(n, ng, 1)
    b = np.asarray(bias16, np.float64).reshape(n, ng, 1)
    return (s * idx.reshape(n, ng, AFFINE_GROUP) + b).reshape(n, d)


def affine_decode_attention(q: np.ndarray, s1: np.ndarray | None, ek: dict, ev: dict,
                            sm_scale: float | None = None, s2: np.ndarray | None = None
                            ) -> np.ndarray:
    """Attention of the G query rows ``q`` [G, d] over the affine-coded tokens of one KV head.

    float64: q_rot = R q (q itself when ``s1`` is None); k_hat, v_hat by
    ``affine_dequantize``;  s_t = scale * (<q_rot, k_hat_t> + sqrt(pi/(2d)) *
    rho16_t * <R2 q_rot, 2 b_t - 1>) (the second term with ``s2``);
    o = softmax(s) v_hat (values are unrotated).  T = 0 gives a zero output.
    """
    q = np.atleast_2d(np.asarray(q, np.float64))
    g, d = q.shape
    if ek["idx"].shape[0] == 0:
        return np.zeros((g, d))
    q_rot = rht_forward(q, s1) if s1 is not None else q
    scores = q_rot @ affine_dequantize(ek["idx"], ek["scale16"], ek["bias16"]).T
    if s2 is not None:
        q_hat = rht_forward(q_rot, s2)
        sgn = 2.0 * np.asarray(ek["sign_bits"], np.float64) - 1.0
        scores = scores + (math.sqrt(math.pi / (2 * d))
                           * np.asarray(ek["rnorm16"], np.float64)[None, :] * (q_hat @ sgn.T))
    scores = default_scale(d, sm_scale) * scores
    p = np.exp(scores - scores.max(axis=-1, keepdims=True))
    vals = affine_dequantize(ev["idx"], ev["scale16"], ev["bias16"])
    return (p @ vals) / p.sum(axis=-1, keepdims=True)


def affine_vector_bytes(d: int, bits: int, qjl: bool = False) -> int:
    """Bytes stored per coded vector: codes, fp16 (scale, bias) per group, and
    with the sketch d/8 sign bytes plus an fp16 residual norm."""
    return bits * d // 8 + 4 * (d // AFFINE_GROUP) + ((d // 8 + 2) if qjl else 0)
