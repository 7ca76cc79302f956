"""GPU parity of tq_quantize_cache (conversion of a dense cache) vs the CPU oracle.

The conversion runs each vector through the same codec as the append, so codes,
sign bits and fp16 norms must equal the oracle's bit for bit.  Covers ragged
rows (empty ones included), a [batch, T, kv_heads, d] cache read in place
through its strides, both lane layouts of the encode kernel (up to 4096 vectors
one vector per warp, above 32 channels per lane), overwriting a non-empty
cache, rows past the capacity, lengths past max_len, and a decode over the
converted cache.
"""
import numpy as np
import pytest
import torch

from tests.tq_helpers import (assert_rows_close, half_bits, oracle_decode_unit, oracle_encode_unit,
                              oracle_tables)

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("turboquant_kv_cache_rht_b200.tq")


def _check_rows(cache, tb, k, v, lengths, qjl, rows=None):
    B, H = k.shape[0], k.shape[1]
    for b in (range(B) if rows is None else rows):
        n = lengths[b]
        for h in range(H):
            ek, ev = oracle_encode_unit(tb, k[b, h, :n], v[b, h, :n])
            assert np.array_equal(cache.k_codes[b, h, :n].cpu().numpy(), ek["codes"]), (b, h)
            assert np.array_equal(cache.v_codes[b, h, :n].cpu().numpy(), ev["codes"]), (b, h)
            assert np.array_equal(half_bits(cache.k_norm, b, h, 0, n), ek["norm16"].view(np.uint16))
            assert np.array_equal(half_bits(cache.v_norm, b, h, 0, n), ev["norm16"].view(np.uint16))
            if qjl:
                assert np.array_equal(cache.k_signs[b, h, :n].cpu().numpy(), ek["signs"])
                assert np.array_equal(half_bits(cache.k_rnorm, b, h, 0, n), ek["rnorm16"].view(np.uint16))


@pytest.mark.parametrize("d,kb,vb,qjl", [(128, 3, 4, False), (128, 3, 4, True), (256, 2, 2, True),
                                         (128, 4, 4, False), (64, 3, 4, True)])
@pytest.mark.parametrize("T,heads_last", [(40, False), (600, False), (600, True)])
def test_convert_ragged_bit_exact(d, kb, vb, qjl, T, heads_last):
    B, H = 3, 4
    g = torch.Generator().manual_seed(d + 10 * kb + vb + qjl + T)
    lengths = [T, 0, T // 3 + 1]
    if heads_last:   # a [batch, T, heads, d] cache, read through its strides
        base = torch.randn(B, T, H, d, generator=g).half()
        kd = base.cuda().permute(0, 2, 1, 3)
        vd = (base * 2).cuda().permute(0, 2, 1, 3)
    else:
        kd = torch.randn(B, H, T, d, generator=g).bfloat16().cuda()
        vd = torch.randn(B, H, T, d, generator=g).bfloat16().cuda()
    cb = tq.Codebook(d, kb, vb, qjl, seed=9)
    cache = tq.Cache(cb, B, H, (T + 15) // 16 * 16, "cuda")
    tq.tq_quantize_cache(cb, cache, kd, vd, torch.tensor(lengths, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert cache.seq_lens.cpu().tolist() == lengths
    assert int(cache.status.item()) == 0
    _check_rows(cache, oracle_tables(d, kb, vb, qjl, 9), kd.cpu(), vd.cpu(), lengths, qjl)


def _convert_raw(cb, cache, kd, vd, lengths, max_len):
    cs = cache.struct()
    lt = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    st = tq.lib.tq_quantize_cache(cb.handle, tq.C.byref(cs), kd.data_ptr(), vd.data_ptr(), 1,
                                  kd.stride(0), kd.stride(1), kd.stride(2), lt.data_ptr(), max_len, None)
    assert st == tq.TQ_OK
    torch.cuda.synchronize()


def test_convert_overwrites_and_flags():
    d, B, H, T = 128, 3, 2, 64
    g = torch.Generator().manual_seed(3)
    cb = tq.Codebook(d, 3, 4, True, seed=1)
    tb = oracle_tables(d, 3, 4, True, 1)
    kd = torch.randn(B, H, T, d, generator=g).bfloat16().cuda()
    vd = torch.randn(B, H, T, d, generator=g).bfloat16().cuda()
    old = torch.randn(B, H, 30, d, generator=g).bfloat16().cuda()

    # a filled cache (30 tokens per row, capacity 48) converted again: row 0 gets
    # 20 tokens (fewer than it held), row 1 asks for 60 > capacity (skipped,
    # untouched), row 2 gets 30
    cache = tq.Cache(cb, B, H, 48, "cuda")
    tq.tq_quantize_append(cb, cache, old, old)
    before = cache.k_codes.clone()
    _convert_raw(cb, cache, kd, vd, [20, 60, 30], 64)
    assert cache.seq_lens.cpu().tolist() == [20, 30, 30]
    assert int(cache.status.item()) == tq.TQ_FLAG_CAPACITY
    assert torch.equal(cache.k_codes[1], before[1])
    _check_rows(cache, tb, kd.cpu(), vd.cpu(), [20, 0, 30], True, rows=(0, 2))

    # lengths past max_len: the first max_len tokens are converted
    cache = tq.Cache(cb, B, H, 48, "cuda")
    _convert_raw(cb, cache, kd, vd, [50, 10, 0], 40)
    assert cache.seq_lens.cpu().tolist() == [40, 10, 0]
    assert int(cache.status.item()) == tq.TQ_FLAG_MAXCTX
    _check_rows(cache, tb, kd.cpu(), vd.cpu(), [40, 10, 0], True)


def test_decode_after_convert():
    d, G, B, H, T = 128, 4, 2, 2, 700
    g = torch.Generator().manual_seed(17)
    kd = torch.randn(B, H, T, d, generator=g).bfloat16()
    vd = torch.randn(B, H, T, d, generator=g).bfloat16()
    q = torch.randn(B, H * G, d, generator=g).bfloat16()
    lengths = [T, 333]
    cb = tq.Codebook(d, 3, 4, True, seed=2)
    cache = tq.Cache(cb, B, H, 704, "cuda")
    tq.tq_quantize_cache(cb, cache, kd.cuda(), vd.cuda(), torch.tensor(lengths, dtype=torch.int32, device="cuda"))
    out = tq.tq_decode_attention(cb, cache, q.cuda(), max_ctx=T).cpu()
    tb = oracle_tables(d, 3, 4, True, 2)
    for b in range(B):
        for h in range(H):
            n = lengths[b]
            ek, ev = oracle_encode_unit(tb, kd[b, h, :n], vd[b, h, :n])
            ref = oracle_decode_unit(tb, q[b, h * G:(h + 1) * G], ek, ev)
            assert_rows_close(out[b, h * G:(h + 1) * G].numpy(), ref, what=f"({b},{h})")
