"""GPU parity of the affine group-64 comparison codec through the C ABI.

"mlx-turboquant" README, "Quantize the KV cache (long-context inference)" and
"How it plugs in": an affine quantized KV cache (group size 64, fp16 scale and
bias) whose keys are rotated, read by an attention that rotates the query.

Encoding (tq_quantize_append in both lane layouts, tq_quantize_cache): codes,
the fp16 (scale, bias) words, sign bits and residual norms must equal the
oracle's bit for bit.  Decode: for every (batch row, query head),
max |gpu - oracle| <= 2e-3 * max |oracle|, the oracle computing in float64 on
its own encoding of the same seeded inputs.  Covers head_dim 64/128/256, every
bit pair, QJL, GQA groups 1-8, ragged lengths (0, 1, tile edges), inputs in
every dtype, exact rounding ties, constant groups, and large common offsets.
"""
import numpy as np
import pytest
import torch

from tests.tq_helpers import (assert_rows_close, half_bits, oracle_decode_unit, oracle_encode_unit,
                              oracle_tables)

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("turboquant_kv_cache_rht_b200.tq")


def _tables(d, kb, vb, qjl, seed):
    return oracle_tables(d, kb, vb, qjl, seed, codebook="affine")


def _codebook(d, kb, vb, qjl, seed):
    return tq.Codebook(d, kb, vb, qjl, seed=seed, codebook="affine")


def _meta_bits(t, b, h, n):
    return t[b, h, :n].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _check_unit(cache, tb, b, h, k_all, v_all, qjl):
    ek, ev = oracle_encode_unit(tb, k_all, v_all)
    n = k_all.shape[0]
    assert np.array_equal(cache.k_codes[b, h, :n].cpu().numpy(), ek["codes"]), "key codes"
    assert np.array_equal(cache.v_codes[b, h, :n].cpu().numpy(), ev["codes"]), "value codes"
    assert np.array_equal(_meta_bits(cache.k_norm, b, h, n), ek["meta16"].view(np.uint16)), "key scale/bias"
    assert np.array_equal(_meta_bits(cache.v_norm, b, h, n), ev["meta16"].view(np.uint16)), "value scale/bias"
    if qjl:
        assert np.array_equal(cache.k_signs[b, h, :n].cpu().numpy(), ek["signs"]), "sign bits"
        assert np.array_equal(half_bits(cache.k_rnorm, b, h, 0, n), ek["rnorm16"].view(np.uint16)), "rnorm"


def _append(cb, B, H, capacity, k, v):
    cache = tq.Cache(cb, B, H, capacity, "cuda")
    tq.tq_quantize_append(cb, cache, k.cuda().contiguous(), v.cuda().contiguous())
    torch.cuda.synchronize()
    return cache


# n = 37 and 700 with B = 2, H = 3 fall on either side of the encoder's switch
# between one vector per warp and 32 channels per lane
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kb,vb", [(2, 2), (2, 3), (3, 4), (4, 4)])
@pytest.mark.parametrize("qjl", [False, True])
@pytest.mark.parametrize("n", [37, 700])
def test_affine_codec_bit_exact(d, kb, vb, qjl, n):
    B, H = 2, 3
    g = torch.Generator().manual_seed(d * 100 + kb * 10 + vb + qjl)
    k = torch.randn(B, H, n, d, generator=g)
    v = torch.randn(B, H, n, d, generator=g) * 3.0 + 0.5
    k[:, :, :, 5] *= 30.0
    v[:, :, :, 9] *= 30.0
    cb = _codebook(d, kb, vb, qjl, 42)
    cache = _append(cb, B, H, (n + 15) // 16 * 16, k, v)
    assert cache.seq_lens.cpu().tolist() == [n] * B and int(cache.status.item()) == 0
    tb = _tables(d, kb, vb, qjl, 42)
    for b in range(B):
        for h in range(H):
            _check_unit(cache, tb, b, h, k[b, h], v[b, h], qjl)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_affine_input_dtypes(dtype):
    d, B, H, n = 128, 1, 2, 40
    g = torch.Generator().manual_seed(5)
    k = torch.randn(B, H, n, d, generator=g).to(dtype)
    v = torch.randn(B, H, n, d, generator=g).to(dtype)
    cache = _append(_codebook(d, 3, 4, True, 3), B, H, 48, k, v)
    for h in range(H):
        _check_unit(cache, _tables(d, 3, 4, True, 3), 0, h, k[0, h], v[0, h], True)


def test_affine_ties_and_constant_groups():
    """Values exactly halfway between two levels (the fp16 scale and bias are
    exact, so (v - bias) / scale lands on k + 1/2 and rounds to even), constant
    groups (scale 0), zero vectors and a single huge channel."""
    d, bits = 128, 3
    lv = (1 << bits) - 1
    rows = []
    for s, b0 in ((0.25, -1.0), (0.125, 0.5), (2.0, -3.0)):
        r = np.empty(d, np.float32)
        for grp in range(d // 64):
            c = np.arange(64) % lv + 0.5            # every tie k + 1/2
            c[0], c[1] = 0, lv                      # the group's min and max on the grid
            r[grp * 64:(grp + 1) * 64] = b0 + s * c
        rows.append(r)
    rows.append(np.full(d, 0.7, np.float32))
    rows.append(np.zeros(d, np.float32))
    one = np.zeros(d, np.float32)
    one[77] = 3e4
    rows.append(one)
    x = torch.from_numpy(np.stack(rows))[None, None]        # [1, 1, 6, d]
    for reps in (1, 300):                                    # both encoder layouts
        xr = x.repeat(1, 1, reps, 1)
        for qjl in (False, True):
            cache = _append(_codebook(d, bits, bits, qjl, 1), 1, 1, (6 * reps + 15) // 16 * 16, xr, xr)
            _check_unit(cache, _tables(d, bits, bits, qjl, 1), 0, 0, xr[0, 0], xr[0, 0], qjl)


def test_affine_convert_matches_append():
    """tq_quantize_cache of a [batch, T, heads, d] cache (read in place through
    its transposed view) with ragged lengths stores what the oracle computes."""
    d, B, H, T = 128, 3, 2, 300
    g = torch.Generator().manual_seed(17)
    k = torch.randn(B, T, H, d, generator=g).bfloat16()
    v = torch.randn(B, T, H, d, generator=g).bfloat16()
    lengths = [300, 1, 129]
    cb = _codebook(d, 4, 4, True, 9)
    cache = tq.Cache(cb, B, H, 304, "cuda")
    kt, vt = k.cuda().transpose(1, 2), v.cuda().transpose(1, 2)
    tq.tq_quantize_cache(cb, cache, kt, vt, torch.tensor(lengths, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert cache.seq_lens.cpu().tolist() == lengths
    tb = _tables(d, 4, 4, True, 9)
    for b in range(B):
        for h in range(H):
            n = lengths[b]
            _check_unit(cache, tb, b, h, k[b, :n, h], v[b, :n, h], True)


def _decode_case(d, kb, vb, qjl, G, lengths, seed, capacity=None, offset=0.0, scale=0.0):
    B, Hkv = len(lengths), 2
    T = max(lengths)
    capacity = capacity or (T + 15) // 16 * 16 or 16
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, Hkv, max(T, 1), d, generator=g)
    v = torch.randn(B, Hkv, max(T, 1), d, generator=g) + offset
    k[..., 3] *= 20.0
    v[..., 9] *= 20.0
    q = torch.randn(B, Hkv * G, d, generator=g)
    for b in range(B):                      # a few keys aligned with a query head
        for h in range(Hkv):
            for t in range(0, lengths[b], 97):
                k[b, h, t] = q[b, h * G + (t % G)] * 1.5
    k, v, q = k.bfloat16(), v.bfloat16(), q.bfloat16()
    cb = _codebook(d, kb, vb, qjl, seed)
    cache = tq.Cache(cb, B, Hkv, capacity, "cuda")
    if T > 0:
        tq.tq_quantize_append(cb, cache, k[:, :, :T].cuda().contiguous(), v[:, :, :T].cuda().contiguous())
    cache.seq_lens.copy_(torch.tensor(lengths, dtype=torch.int32))
    out = tq.tq_decode_attention(cb, cache, q.cuda(), softmax_scale=scale, max_ctx=capacity)
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    tb = _tables(d, kb, vb, qjl, seed)
    ref = np.zeros((B, Hkv * G, d))
    for b in range(B):
        for h in range(Hkv):
            n = lengths[b]
            ek, ev = oracle_encode_unit(tb, k[b, h, :n], v[b, h, :n])
            ref[b, h * G:(h + 1) * G] = oracle_decode_unit(tb, q[b, h * G:(h + 1) * G], ek, ev,
                                                           scale if scale > 0 else None)
    assert_rows_close(out.cpu().numpy().reshape(-1, d), ref.reshape(-1, d))
    return out


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kb,vb,qjl", [(4, 4, False), (3, 4, True), (2, 2, True), (2, 3, False),
                                       (3, 3, False)])
def test_affine_decode_matches_oracle(d, kb, vb, qjl):
    _decode_case(d, kb, vb, qjl, 4, [300, 129], seed=kb * 10 + vb + 100 * qjl)


@pytest.mark.parametrize("G", [1, 2, 8])
@pytest.mark.parametrize("qjl", [False, True])
def test_affine_decode_groups_and_ragged_rows(G, qjl):
    _decode_case(128, 4, 4, qjl, G, [517, 1, 0, 64, 65], seed=50 + G)


def test_affine_decode_offsets_and_scale():
    """Values far from zero (the bias carries them) and a custom softmax scale."""
    _decode_case(128, 4, 4, False, 4, [700, 250], seed=61, offset=6.0)
    _decode_case(256, 3, 4, True, 2, [333], seed=62, scale=0.05)


def test_affine_decode_partition_independent():
    """The same cache decoded with a larger max_ctx (another work partition)
    gives the same result to rounding."""
    d, G = 128, 4
    out1 = _decode_case(d, 4, 4, False, G, [1500, 40], seed=71, capacity=1504)
    out2 = _decode_case(d, 4, 4, False, G, [1500, 40], seed=71, capacity=4096)
    assert torch.allclose(out1, out2, rtol=0, atol=2e-3 * float(out1.abs().max()))
