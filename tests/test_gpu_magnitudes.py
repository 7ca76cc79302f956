"""GPU decode parity across value and key magnitudes (through the C ABI).

The decode folds each token's fp16 value norm into its softmax weight and
feeds the product to the tensor cores in fp16 parts, and it scales the key
scores by the fp16 key norms.  These tests put the norms far from 1 -- tiny
(fp16 subnormal) and large -- and mix them inside one row, with all-zero value
vectors, with and without the QJL sketch, at every head dim, for the Lloyd-Max
and the affine codecs.  The bar is the decode's: per (batch row, query head),
max |gpu - oracle| <= 2e-3 * max |oracle| ("TurboQuant Performance Benefits
...", "What Is TurboQuant?": attention over the compressed cache; "mlx-turboquant"
README, "The 1-bit QJL residual").

The largest scales keep every norm below fp16's 65504 (a larger norm is stored
as an infinite fp16 norm, which the codec documents as undefined).
"""
import numpy as np
import pytest
import torch

from tests.tq_helpers import assert_rows_close, oracle_decode_unit, oracle_encode_unit, oracle_tables

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("turboquant_kv_cache_rht_b200.tq")


def _run(d, kb, vb, qjl, lengths, G, k, v, q, seed, codebook="gaussian"):
    B, Hkv = k.shape[0], k.shape[1]
    cap = (max(lengths) + 15) // 16 * 16
    cb = tq.Codebook(d, kb, vb, qjl, seed=seed, codebook=codebook)
    cache = tq.Cache(cb, B, Hkv, cap, "cuda")
    tq.tq_quantize_append(cb, cache, k.cuda(), v.cuda())
    cache.seq_lens.copy_(torch.tensor(lengths, dtype=torch.int32))
    out = tq.tq_decode_attention(cb, cache, q.cuda(), max_ctx=cap).cpu().numpy()
    tb = oracle_tables(d, kb, vb, qjl, seed, codebook=codebook)
    for b in range(B):
        for h in range(Hkv):
            n = lengths[b]
            ek, ev = oracle_encode_unit(tb, k[b, h, :n], v[b, h, :n])
            ref = oracle_decode_unit(tb, q[b, h * G:(h + 1) * G], ek, ev)
            assert np.isfinite(out[b, h * G:(h + 1) * G]).all()
            assert_rows_close(out[b, h * G:(h + 1) * G], ref, what=f"({b},{h})")
    return out


def _inputs(d, B, Hkv, G, T, seed, v_scale=1.0, k_scale=1.0):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, Hkv, T, d, generator=g) * k_scale
    v = torch.randn(B, Hkv, T, d, generator=g) * v_scale
    q = torch.randn(B, Hkv * G, d, generator=g)
    return k, v, q


def _max_scale(d):
    # N(0,1) vectors: ||x|| ~ sqrt(d) (at most ~1.3 sqrt(d) over these sizes)
    return 4.0e4 / (1.3 * np.sqrt(d))


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("qjl", [False, True])
@pytest.mark.parametrize("v_scale", [1e-6, 1e-4, 1e-2, 1e2, "max"])
def test_value_scales(d, qjl, v_scale):
    if v_scale == "max":
        v_scale = _max_scale(d)
    G, B, Hkv = 4, 2, 2
    lengths = [300, 77]
    k, v, q = _inputs(d, B, Hkv, G, 300, seed=int(d + 7 * qjl), v_scale=v_scale)
    _run(d, 3, 4, qjl, lengths, G, k.float(), v.float(), q.float(), seed=5)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("qjl", [False, True])
@pytest.mark.parametrize("k_scale", [1e-6, 1e-3, 1e2])
def test_key_scales(d, qjl, k_scale):
    # keys far from unit norm: the scores shrink to ~0 (uniform softmax) or
    # grow large (one token dominates); the query is scaled back so that the
    # logits stay moderate at 1e2
    G, B, Hkv = 4, 1, 2
    lengths = [250]
    k, v, q = _inputs(d, B, Hkv, G, 250, seed=int(3 * d + qjl), k_scale=k_scale)
    if k_scale > 1:
        q = q / k_scale
    _run(d, 2, 3, qjl, lengths, G, k.float(), v.float(), q.float(), seed=6)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("qjl", [False, True])
def test_mixed_norms_and_zero_values(d, qjl):
    # one row mixes tokens whose values are ~1e-6, ~1, ~1e2 and exactly zero,
    # in runs that straddle the 16-token slabs and 64-token tiles; the other
    # row holds only zero values (its output is exactly zero)
    G, B, Hkv, T = 4, 2, 2, 400
    k, v, q = _inputs(d, B, Hkv, G, T, seed=90 + d + qjl)
    scale = torch.ones(T)
    scale[0:40] = 1e-6
    scale[40:70] = 0.0
    scale[70:75] = 1e2
    scale[150:260] = 1e-4
    scale[300:301] = 0.0
    scale[333:390] = 3e-5
    v[0] *= scale[None, :, None]
    v[1] = 0.0
    out = _run(d, 3, 4, qjl, [T, 200], G, k.float(), v.float(), q.float(), seed=8)
    assert np.all(out[1] == 0.0)


@pytest.mark.parametrize("G", [1, 8])
def test_tiny_values_gqa_groups(G):
    d, B, Hkv = 128, 1, 2
    k, v, q = _inputs(d, B, Hkv, G, 333, seed=70 + G, v_scale=2e-6)
    _run(d, 3, 4, True, [333], G, k.float(), v.float(), q.float(), seed=9)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("v_scale", [1e-6, 1e-3, 1e2])
def test_affine_value_scales(d, v_scale):
    G, B, Hkv = 4, 1, 2
    k, v, q = _inputs(d, B, Hkv, G, 260, seed=40 + d, v_scale=v_scale)
    v[0, 0, 100:130] = 0.0
    _run(d, 4, 4, False, [260], G, k.float(), v.float(), q.float(), seed=10, codebook="affine")
