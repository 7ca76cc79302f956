"""The decode entry point that allocates nothing (GPU).

Some callers cannot allocate device memory, so they cannot pass the workspace
tq_decode_attention needs; tq_decode_attention_noalloc uses a static scratch
array inside the library instead.  This test calls it through the C ABI twice
in a row, on different inputs, and checks each result against the CPU oracle
on the same seeded inputs (per row within the decode tolerance) and against
tq_decode_attention with a caller workspace (the two share the same kernels,
so they agree exactly in practice).  It also checks the size limit.  It builds
its own inputs, so it passes alone in a fresh process as well as after other
tests.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from tests.tq_helpers import assert_rows_close, oracle_decode_unit, oracle_encode_unit, oracle_tables

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("turboquant_kv_cache_rht_b200.tq")


def _raw_kv(batch, kv_heads, length, d, seed):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(batch, kv_heads, length, d, generator=g).bfloat16()
    v = torch.randn(batch, kv_heads, length, d, generator=g).bfloat16()
    return k, v


def _filled_cache(cb, k, v, capacity):
    cache = tq.Cache(cb, k.shape[0], k.shape[1], capacity, "cuda")
    tq.tq_quantize_append(cb, cache, k.cuda(), v.cuda())
    return cache


def _oracle(tb, k, v, q, G):
    out = np.zeros(q.shape, np.float64)
    for b in range(k.shape[0]):
        for h in range(k.shape[1]):
            ek, ev = oracle_encode_unit(tb, k[b, h], v[b, h])
            out[b, h * G:(h + 1) * G] = oracle_decode_unit(tb, q[b, h * G:(h + 1) * G], ek, ev)
    return out


def _noalloc(cb, cache, q, out, max_ctx):
    cs = cache.struct()
    st = tq.lib.tq_decode_attention_noalloc(cb.handle, C.byref(cs), q.data_ptr(), 1, q.shape[1],
                                            0.0, max_ctx, out.data_ptr(),
                                            torch.cuda.current_stream().cuda_stream)
    assert st == tq.TQ_OK, tq.tq_last_error()
    return out


@pytest.mark.parametrize("d,kb,vb,qjl,codebook", [
    (128, 3, 4, True, "gaussian"),     # the QJL sketch
    (128, 3, 4, False, "gaussian"),
    (128, 4, 4, False, "affine"),      # the affine comparison codec
    (256, 2, 2, True, "gaussian"),     # head_dim 256, 2-bit codes
])
def test_noalloc_matches_oracle_twice(d, kb, vb, qjl, codebook):
    cb = tq.Codebook(d, kb, vb, qjl=qjl, seed=3, codebook=codebook)
    tb = oracle_tables(d, kb, vb, qjl, 3, codebook=codebook)
    cases = [(2, 4, 4, 1000, 1024, 11), (1, 8, 2, 3000, 3008, 12)]   # two calls in a row
    for batch, kv_heads, group, length, cap, seed in cases:
        assert tq.tq_decode_workspace_bytes(cb, batch, kv_heads * group, kv_heads, cap) <= (8 << 20)
        k, v = _raw_kv(batch, kv_heads, length, d, seed)
        cache = _filled_cache(cb, k, v, cap)
        g = torch.Generator().manual_seed(seed + 100)
        q = torch.randn(batch, kv_heads * group, d, generator=g).bfloat16()
        out = torch.full((batch, kv_heads * group, d), float("nan"), device="cuda")
        got = _noalloc(cb, cache, q.cuda(), out, cap).clone()
        ref = tq.tq_decode_attention(cb, cache, q.cuda(), max_ctx=cap)
        torch.cuda.synchronize()
        assert torch.isfinite(got).all()
        got = got.cpu().numpy().reshape(-1, d)
        assert_rows_close(got, _oracle(tb, k, v, q, group).reshape(-1, d), what="oracle")
        assert_rows_close(got, ref.cpu().numpy().reshape(-1, d), what="workspace entry point")


def test_noalloc_rejects_decodes_larger_than_its_scratch():
    cb = tq.Codebook(256, 2, 2, qjl=False, seed=0)
    # find a batch whose split partials need more than the 8 MiB static scratch
    batch = next(bt for bt in (64, 128, 256, 512, 1024)
                 if tq.tq_decode_workspace_bytes(cb, bt, 64, 8, 65536) > (8 << 20))
    cache = tq.Cache(cb, batch, 8, 16, "cuda")
    q = torch.zeros(batch, 64, 256, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(batch, 64, 256, device="cuda")
    cs = cache.struct()
    cs.capacity = 65536   # sizes only: the call is rejected before any launch
    st = tq.lib.tq_decode_attention_noalloc(cb.handle, C.byref(cs), q.data_ptr(), 1, 64, 0.0,
                                            65536, out.data_ptr(), None)
    assert st == tq.TQ_ERR_CAPACITY
    assert "scratch" in tq.tq_last_error()
    assert np.all(out.cpu().numpy() == 0)
