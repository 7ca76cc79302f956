"""Guard-byte tests (GPU): no kernel writes outside the buffers it is given.

Every device buffer a call writes -- the cache arrays, seq_lens, status,
append_sync, the decode output and workspace, the weights' codes and norms, the
matmul output and workspace -- is carved out of a larger allocation whose
leading and trailing guard regions are filled with a byte pattern.  The calls
run on edge shapes (head_dim 64 with 3-bit codes, whose 24-byte rows are
staged in 8-byte pieces; partial last tiles; rows filled to exactly the
capacity; an append past the capacity; max_ctx below a row's length; ragged
and empty rows; a workspace of exactly the size the library asks for), then
every guard byte must still hold the pattern.  The results are also compared
with the same calls on ordinary (unguarded) buffers, so the guarded runs are
real work.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("turboquant_kv_cache_rht_b200.tq")

GUARD = 4096          # bytes on each side (keeps every payload 16-byte aligned)
PATTERN = 0xA5


class Guarded:
    """Device buffers with guard regions; `view` hands out the payloads."""

    def __init__(self):
        self.bufs = []

    def view(self, shape, dtype, fill=0):
        esz = torch.empty((), dtype=dtype).element_size()
        n = int(np.prod(shape)) * esz
        buf = torch.full((GUARD + n + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        payload = buf[GUARD:GUARD + n]
        payload.fill_(fill)
        self.bufs.append((buf, n))
        return payload.view(dtype).view(*shape)

    def check(self, what=""):
        torch.cuda.synchronize()
        for i, (buf, n) in enumerate(self.bufs):
            lo = buf[:GUARD].cpu().numpy()
            hi = buf[GUARD + n:].cpu().numpy()
            assert np.all(lo == PATTERN), f"{what}: buffer {i} leading guard overwritten"
            assert np.all(hi == PATTERN), f"{what}: buffer {i} trailing guard overwritten"


class GuardedCache(tq.Cache):
    """tq.Cache whose arrays sit between guard regions."""

    def __init__(self, cb, batch, kv_heads, capacity, g: Guarded):
        lay = cb.layout
        n = (batch, kv_heads, capacity)
        self.batch, self.kv_heads, self.capacity = batch, kv_heads, capacity
        self.k_codes = g.view((*n, lay.k_code_bytes), torch.uint8)
        self.v_codes = g.view((*n, lay.v_code_bytes), torch.uint8)
        self.k_signs = g.view((*n, lay.k_sign_bytes), torch.uint8) if cb.qjl else None
        nh = (lay.norm_halves,) if cb.affine else ()
        self.k_norm = g.view((*n, *nh), torch.float16)
        self.v_norm = g.view((*n, *nh), torch.float16)
        self.k_rnorm = g.view(n, torch.float16) if cb.qjl else None
        self.seq_lens = g.view((batch,), torch.int32)
        self.status = g.view((1,), torch.int32)
        self.append_sync = g.view((batch,), torch.int32)


SHAPES = [  # head_dim, k_bits, v_bits, qjl, codebook
    (64, 3, 4, True, "gaussian"),
    (64, 3, 3, False, "gaussian"),
    (128, 3, 4, False, "gaussian"),
    (128, 2, 3, True, "gaussian"),
    (256, 2, 2, True, "gaussian"),
    (256, 4, 4, False, "gaussian"),
    (128, 4, 4, True, "affine"),
    (64, 3, 4, False, "affine"),
]


def _kv(batch, heads, n, d, seed):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(batch, heads, n, d, generator=g).bfloat16().cuda()
    v = torch.randn(batch, heads, n, d, generator=g).bfloat16().cuda()
    return k, v


def _same_cache(a, b):
    for name in ("k_codes", "v_codes", "k_signs", "k_norm", "v_norm", "k_rnorm", "seq_lens"):
        x, y = getattr(a, name), getattr(b, name)
        if x is not None:
            assert torch.equal(x, y), name


@pytest.mark.parametrize("d,kb,vb,qjl,codebook", SHAPES)
def test_append_and_decode_stay_in_bounds(d, kb, vb, qjl, codebook):
    cb = tq.Codebook(d, kb, vb, qjl, seed=21, codebook=codebook)
    B, H, G, cap = 3, 2, 4, 80
    g = Guarded()
    cache = GuardedCache(cb, B, H, cap, g)
    plain = tq.Cache(cb, B, H, cap, "cuda")
    # appends of 17, 46 and 17 tokens fill every row to exactly `capacity`;
    # a fourth append passes it, is skipped and sets the capacity flag
    for i, n in enumerate((17, 46, 17, 5)):
        k, v = _kv(B, H, n, d, 100 + i)
        tq.tq_quantize_append(cb, cache, k, v)
        tq.tq_quantize_append(cb, plain, k, v)
    g.check("append")
    assert int(cache.status.item()) & tq.TQ_FLAG_CAPACITY
    _same_cache(cache, plain)
    assert cache.seq_lens.tolist() == [cap] * B
    # ragged rows: full, a partial last tile, empty
    lens = torch.tensor([cap, 37, 0], dtype=torch.int32)
    cache.seq_lens.copy_(lens)
    plain.seq_lens.copy_(lens)
    q = torch.randn(B, H * G, d, generator=torch.Generator().manual_seed(7)).bfloat16().cuda()
    for max_ctx in (cap, 48):      # 48 < 80: the first row's tail is cut and flagged
        need = tq.tq_decode_workspace_bytes(cb, B, H * G, H, max_ctx)
        ws = g.view((need,), torch.uint8)
        out = g.view((B, H * G, d), torch.float32)
        cache.status.zero_()
        tq.tq_decode_attention(cb, cache, q, out=out, max_ctx=max_ctx, workspace=ws)
        ref = tq.tq_decode_attention(cb, plain, q, max_ctx=max_ctx)
        g.check(f"decode max_ctx {max_ctx}")
        assert torch.equal(out, ref)
        assert torch.all(out[2] == 0)
        flagged = bool(int(cache.status.item()) & tq.TQ_FLAG_MAXCTX)
        assert flagged == (max_ctx < cap)
        assert not int(cache.status.item()) & tq.TQ_FLAG_LAYOUT


@pytest.mark.parametrize("d,kb,vb,qjl,codebook", SHAPES[:5] + SHAPES[6:7])
def test_convert_stays_in_bounds(d, kb, vb, qjl, codebook):
    cb = tq.Codebook(d, kb, vb, qjl, seed=22, codebook=codebook)
    B, H, cap, T = 4, 2, 64, 70
    g = Guarded()
    cache = GuardedCache(cb, B, H, cap, g)
    plain = tq.Cache(cb, B, H, cap, "cuda")
    # a [batch, T, heads, d] dense cache read in place through its strides
    gen = torch.Generator().manual_seed(5)
    k = torch.randn(B, T, H, d, generator=gen).bfloat16().cuda().transpose(1, 2)
    v = torch.randn(B, T, H, d, generator=gen).bfloat16().cuda().transpose(1, 2)
    # exactly capacity, a partial tile, zero, and one past capacity (skipped, flagged)
    lengths = g.view((B,), torch.int32)
    lengths.copy_(torch.tensor([cap, 33, 0, cap + 1], dtype=torch.int32))
    tq.tq_quantize_cache(cb, cache, k, v, lengths=lengths)
    tq.tq_quantize_cache(cb, plain, k, v, lengths=lengths.clone())
    g.check("convert")
    _same_cache(cache, plain)
    assert int(cache.status.item()) & tq.TQ_FLAG_CAPACITY


@pytest.mark.parametrize("bits,m", [(2, 1), (3, 5), (4, 16)])
def test_lut_matmul_stays_in_bounds(bits, m):
    d, rows, k = 128, 272, 768
    cb = tq.Codebook(d, bits, bits, seed=9)
    gen = torch.Generator().manual_seed(bits)
    w = torch.randn(rows, k, generator=gen).bfloat16().cuda()
    x = torch.randn(m, k, generator=gen).bfloat16().cuda()
    g = Guarded()
    nb = k // d
    codes = g.view((nb, rows, cb.layout.k_code_bytes), torch.uint8)
    norms = g.view((nb, rows), torch.float16)
    st = tq.lib.tq_weights_quantize(cb.handle, w.data_ptr(), 1, rows, k, codes.data_ptr(),
                                    norms.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == tq.TQ_OK, tq.tq_last_error()
    nbytes = tq.tq_lut_matmul_workspace_bytes(cb, rows, k, m)
    ws = g.view((max(nbytes, 16),), torch.uint8)
    y = g.view((m, rows), torch.float32)
    st = tq.lib.tq_lut_matmul(cb.handle, codes.data_ptr(), norms.data_ptr(), rows, k, x.data_ptr(), 1,
                              m, y.data_ptr(), ws.data_ptr(), nbytes,
                              torch.cuda.current_stream().cuda_stream)
    assert st == tq.TQ_OK, tq.tq_last_error()
    g.check("lut matmul")
    ref = tq.QuantizedWeights(cb, w)
    assert torch.equal(codes, ref.codes) and torch.equal(norms, ref.norms)
    assert torch.equal(y, ref.matmul(x))
