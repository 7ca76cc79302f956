"""GPU codec parity: tq_quantize_append through the C ABI vs the CPU oracle.

Codes, sign bits and fp16 norms must be bit-identical.  Covers head_dim 128 and
256, every bit width, QJL on/off, fp32/bf16/fp16 inputs, several appends in a
row, ragged appends, adversarial vectors (zero, +-0, huge outliers, subnormals,
all energy in one rotated coordinate), capacity overflow (flag, row skipped).
"""
import numpy as np
import pytest
import torch

import oracle as o
from tests.tq_helpers import half_bits, oracle_encode_unit, oracle_tables

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("turboquant_kv_cache_rht_b200.tq")


def _run(cb, batch, kv_heads, capacity, chunks, device="cuda"):
    """Append the list of (k, v) chunks [B, H, n, d] in order; returns the cache."""
    cache = tq.Cache(cb, batch, kv_heads, capacity, device)
    for k, v in chunks:
        tq.tq_quantize_append(cb, cache, k.to(device).contiguous(), v.to(device).contiguous())
    torch.cuda.synchronize()
    return cache


def _check_unit(cache, tb, b, h, k_all, v_all, qjl):
    ek, ev = oracle_encode_unit(tb, k_all, v_all)
    n = k_all.shape[0]
    assert np.array_equal(cache.k_codes[b, h, :n].cpu().numpy(), ek["codes"]), "key codes"
    assert np.array_equal(cache.v_codes[b, h, :n].cpu().numpy(), ev["codes"]), "value codes"
    assert np.array_equal(half_bits(cache.k_norm, b, h, 0, n), ek["norm16"].view(np.uint16)), "key norms"
    assert np.array_equal(half_bits(cache.v_norm, b, h, 0, n), ev["norm16"].view(np.uint16)), "value norms"
    if qjl:
        assert np.array_equal(cache.k_signs[b, h, :n].cpu().numpy(), ek["signs"]), "sign bits"
        assert np.array_equal(half_bits(cache.k_rnorm, b, h, 0, n),
                              ek["rnorm16"].view(np.uint16)), "residual norms"


# The encode kernel has two lane layouts, chosen by the append's total vector
# count (keys and values of every row): up to 4096 vectors one vector per warp,
# above that 32 channels per lane.  n = 37 and n = 700 (with B = 2, H = 3) fall
# on either side, so every case runs through both.
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kb,vb", [(2, 2), (2, 3), (3, 3), (3, 4), (4, 4)])
@pytest.mark.parametrize("qjl", [False, True])
@pytest.mark.parametrize("n", [37, 700])
def test_codec_bit_exact(d, kb, vb, qjl, n):
    B, H = 2, 3
    assert (2 * B * H * n > 4096) == (n == 700)
    g = torch.Generator().manual_seed(d * 100 + kb * 10 + vb + qjl)
    k = torch.randn(B, H, n, d, generator=g)
    v = torch.randn(B, H, n, d, generator=g) * 3.0
    k[:, :, :, 5] *= 30.0                      # outlier channel
    cb = tq.Codebook(d, kb, vb, qjl, seed=42)
    tb = oracle_tables(d, kb, vb, qjl, 42)
    cache = _run(cb, B, H, (n + 15) // 16 * 16, [(k, v)])
    assert cache.seq_lens.cpu().tolist() == [n] * B
    assert cache.append_sync.cpu().tolist() == [0] * B
    assert int(cache.status.item()) == 0
    for b in range(B):
        for h in range(H):
            _check_unit(cache, tb, b, h, k[b, h], v[b, h], qjl)


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("kb,vb,qjl", [(2, 2, True), (3, 4, False), (4, 4, True)])
@pytest.mark.parametrize("n", [37, 700])
def test_codec_bit_exact_sphere_codebook(d, kb, vb, qjl, n):
    """The codec with the head_dim-specific sphere codebook (both lane layouts)."""
    B, H = 2, 3
    g = torch.Generator().manual_seed(7 * d + kb + n)
    k = torch.randn(B, H, n, d, generator=g).bfloat16()
    v = torch.randn(B, H, n, d, generator=g).bfloat16()
    cb = tq.Codebook(d, kb, vb, qjl, seed=5, codebook="sphere")
    tb = oracle_tables(d, kb, vb, qjl, 5, codebook="sphere")
    cache = _run(cb, B, H, (n + 15) // 16 * 16, [(k, v)])
    for b in range(B):
        for h in range(H):
            _check_unit(cache, tb, b, h, k[b, h], v[b, h], qjl)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_input_dtypes(dtype):
    d, B, H, n = 128, 1, 2, 16
    g = torch.Generator().manual_seed(5)
    k = torch.randn(B, H, n, d, generator=g).to(dtype)
    v = torch.randn(B, H, n, d, generator=g).to(dtype)
    cb = tq.Codebook(d, 3, 4, True, seed=3)
    cache = _run(cb, B, H, 16, [(k, v)])
    tb = oracle_tables(d, 3, 4, True, 3)
    for h in range(H):
        _check_unit(cache, tb, 0, h, k[0, h], v[0, h], True)


def test_repeated_and_ragged_appends():
    d, B, H = 128, 3, 2
    g = torch.Generator().manual_seed(9)
    chunks = [(torch.randn(B, H, n, d, generator=g).bfloat16(),
               torch.randn(B, H, n, d, generator=g).bfloat16()) for n in (5, 1, 1, 17, 1)]
    cb = tq.Codebook(d, 2, 3, True, seed=11)
    cache = _run(cb, B, H, 32, chunks)
    assert cache.seq_lens.cpu().tolist() == [25] * B
    tb = oracle_tables(d, 2, 3, True, 11)
    k_all = torch.cat([c[0] for c in chunks], dim=2)
    v_all = torch.cat([c[1] for c in chunks], dim=2)
    for b in range(B):
        for h in range(H):
            _check_unit(cache, tb, b, h, k_all[b, h], v_all[b, h], True)


def test_adversarial_vectors():
    d, H = 256, 1
    s1 = o.rotation_signs(0, d)
    rows = [torch.zeros(d), -torch.zeros(d), torch.full((d,), 1e-40),   # subnormals
            torch.from_numpy(s1.astype(np.float32)) * 0.25,            # all energy on channel 0
            torch.nn.functional.one_hot(torch.tensor(7), d).float() * 3e4,
            torch.linspace(-1000, 1000, d), torch.randn(d, generator=torch.Generator().manual_seed(1)) * 1e-20]
    k = torch.stack(rows)[None, None]                  # [1, 1, n, d]
    v = torch.flip(k, dims=[2]).contiguous()
    # the 7 rows alone (one vector per warp), and repeated 300 times (4200
    # vectors: 32 channels per lane)
    for reps in (1, 300):
        kr, vr = k.repeat(1, 1, reps, 1), v.repeat(1, 1, reps, 1)
        for qjl in (False, True):
            for kb, vb in ((2, 2), (3, 4), (4, 4)):
                cb = tq.Codebook(d, kb, vb, qjl, seed=0)
                cache = _run(cb, 1, H, (7 * reps + 15) // 16 * 16, [(kr, vr)])
                _check_unit(cache, oracle_tables(d, kb, vb, qjl, 0), 0, 0, kr[0, 0], vr[0, 0], qjl)


def test_capacity_overflow_flags_and_skips():
    d, B, H = 128, 2, 1
    cb = tq.Codebook(d, 3, 4)
    cache = tq.Cache(cb, B, H, 16, "cuda")
    cache.seq_lens.copy_(torch.tensor([10, 3], dtype=torch.int32))
    k = torch.randn(B, H, 8, d, device="cuda")
    before = cache.k_codes.clone()
    tq.tq_quantize_append(cb, cache, k, k.clone())
    torch.cuda.synchronize()
    assert cache.seq_lens.cpu().tolist() == [10, 11]      # row 0 would reach 18 > 16
    assert int(cache.status.item()) & tq.TQ_FLAG_CAPACITY
    assert torch.equal(cache.k_codes[0], before[0])       # row 0 untouched
    assert not torch.equal(cache.k_codes[1, 0, 3:11], before[1, 0, 3:11])
    assert cache.append_sync.cpu().tolist() == [0, 0]


def test_many_blocks_per_row():
    """A bulk append spreads one batch row over many blocks; the length is
    published once, after every block wrote."""
    d, B, H, n = 128, 2, 8, 700
    g = torch.Generator().manual_seed(21)
    k = torch.randn(B, H, n, d, generator=g).bfloat16()
    v = torch.randn(B, H, n, d, generator=g).bfloat16()
    cb = tq.Codebook(d, 3, 4, True, seed=5)
    cache = _run(cb, B, H, 704, [(k, v)])
    assert cache.seq_lens.cpu().tolist() == [n, n]
    tb = oracle_tables(d, 3, 4, True, 5)
    for b, h in ((0, 0), (1, 7), (0, 5)):
        _check_unit(cache, tb, b, h, k[b, h], v[b, h], True)
