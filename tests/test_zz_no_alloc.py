"""The decode entry point that allocates nothing (GPU).

Some callers cannot allocate device memory, so they cannot pass the workspace
tq_decode_attention needs; tq_decode_attention_noalloc uses a static scratch
array inside the library instead.  This test calls it through the C ABI twice
in a row, on different inputs, and checks each result against
tq_decode_attention with a caller workspace, within the decode tolerance the
other tests use (the two share the same kernels, so the results agree
exactly in practice).  It also checks the size limit.  It builds its own
inputs, so it passes alone in a fresh process as well as after other tests.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from tests.tq_helpers import assert_rows_close

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("turboquant_kv_cache_rht_b200.tq")


def _filled_cache(cb, batch, kv_heads, length, capacity, seed):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(batch, kv_heads, length, cb.head_dim, generator=g).bfloat16().cuda()
    v = torch.randn(batch, kv_heads, length, cb.head_dim, generator=g).bfloat16().cuda()
    cache = tq.Cache(cb, batch, kv_heads, capacity, "cuda")
    tq.tq_quantize_append(cb, cache, k, v)
    return cache


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
def test_noalloc_matches_workspace_entry_point_twice(d, kb, vb, qjl, codebook):
    cb = tq.Codebook(d, kb, vb, qjl=qjl, seed=3, codebook=codebook)
    cases = [(2, 4, 4, 1000, 1024, 11), (1, 8, 2, 3000, 3008, 12)]   # two calls in a row
    for batch, kv_heads, group, length, cap, seed in cases:
        assert tq.tq_decode_workspace_bytes(cb, batch, kv_heads * group, kv_heads, cap) <= (8 << 20)
        cache = _filled_cache(cb, batch, kv_heads, length, cap, seed)
        g = torch.Generator().manual_seed(seed + 100)
        q = torch.randn(batch, kv_heads * group, d, generator=g).bfloat16().cuda()
        out = torch.full((batch, kv_heads * group, d), float("nan"), device="cuda")
        got = _noalloc(cb, cache, q, out, cap).clone()
        ref = tq.tq_decode_attention(cb, cache, q, max_ctx=cap)
        torch.cuda.synchronize()
        assert torch.isfinite(got).all()
        assert_rows_close(got.cpu().numpy().reshape(-1, d), ref.cpu().numpy().reshape(-1, d))


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
