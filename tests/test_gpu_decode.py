"""GPU decode parity: tq_decode_attention through the C ABI vs the CPU oracle.

The oracle encodes the same seeded raw K/V itself (codes are bit-exact, see
test_gpu_codec) and computes attention in float64; the GPU result must satisfy,
for every (batch row, query head), max |gpu - oracle| <= 2e-3 * max |oracle|.
Covers several tiles plus a ragged tail, lengths 0/1/127/128/129, all GQA
groups, both head dims, every bit pair, QJL, custom softmax scale, repeat-run
determinism, independence of the work partition, and the max_ctx flag.
"""
import numpy as np
import pytest
import torch

from tests.tq_helpers import assert_rows_close, oracle_decode_unit, oracle_encode_unit, oracle_tables

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("turboquant_kv_cache_rht_b200.tq")


def _setup(d, kb, vb, qjl, B, Hkv, G, lengths, capacity, seed=7, dtype=torch.bfloat16,
           corr=False):
    g = torch.Generator().manual_seed(seed)
    T = max(lengths)
    k = torch.randn(B, Hkv, T, d, generator=g)
    v = torch.randn(B, Hkv, T, d, generator=g)
    k[..., 3] *= 20.0
    v[..., 9] *= 20.0
    q = torch.randn(B, Hkv * G, d, generator=g)
    if corr:   # a few keys strongly aligned with a query head: peaked softmax
        for b in range(B):
            for h in range(Hkv):
                for t in range(0, lengths[b], 97):
                    k[b, h, t] = q[b, h * G + (t % G)] * 1.5
    k, v, q = k.to(dtype), v.to(dtype), q.to(dtype)
    cb = tq.Codebook(d, kb, vb, qjl, seed=seed)
    cache = tq.Cache(cb, B, Hkv, capacity, "cuda")
    # append the longest length for every row, then shorten rows to their own
    # length: decode attends only slots below seq_lens[b]
    if T > 0:
        tq.tq_quantize_append(cb, cache, k.cuda(), v.cuda())
    cache.seq_lens.copy_(torch.tensor(lengths, dtype=torch.int32))
    torch.cuda.synchronize()
    return cb, cache, k, v, q


def _oracle(d, kb, vb, qjl, seed, k, v, q, lengths, G, scale=None):
    tb = oracle_tables(d, kb, vb, qjl, seed)
    B, Hkv = k.shape[0], k.shape[1]
    out = np.zeros((B, Hkv * G, d))
    for b in range(B):
        for h in range(Hkv):
            n = lengths[b]
            ek, ev = oracle_encode_unit(tb, k[b, h, :n], v[b, h, :n])
            out[b, h * G:(h + 1) * G] = oracle_decode_unit(tb, q[b, h * G:(h + 1) * G], ek, ev, scale)
    return out


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kb,vb,qjl", [(3, 4, False), (3, 4, True), (2, 2, True), (4, 4, False),
                                       (2, 3, False), (3, 3, True), (2, 2, False), (3, 3, False)])
def test_decode_matches_oracle(d, kb, vb, qjl):
    G, B, Hkv = 4, 2, 2
    lengths = [300, 129]
    cb, cache, k, v, q = _setup(d, kb, vb, qjl, B, Hkv, G, lengths, 320, seed=kb * 10 + vb)
    out = tq.tq_decode_attention(cb, cache, q.cuda(), max_ctx=320)
    torch.cuda.synchronize()
    ref = _oracle(d, kb, vb, qjl, kb * 10 + vb, k, v, q, lengths, G)
    assert_rows_close(out.cpu().numpy().reshape(-1, d), ref.reshape(-1, d))


@pytest.mark.parametrize("G", [1, 8])
@pytest.mark.parametrize("qjl", [False, True])
def test_gqa_groups_head_dim_64(G, qjl):
    d, B, Hkv = 64, 2, 2
    lengths = [517, 64]
    cb, cache, k, v, q = _setup(d, 3, 4, qjl, B, Hkv, G, lengths, 528, seed=40 + G, corr=True)
    out = tq.tq_decode_attention(cb, cache, q.cuda(), max_ctx=528)
    torch.cuda.synchronize()
    ref = _oracle(d, 3, 4, qjl, 40 + G, k, v, q, lengths, G)
    assert_rows_close(out.cpu().numpy().reshape(-1, d), ref.reshape(-1, d))


# Every group size on the table layouts of head_dim 128: 3-bit keys / 4-bit
# values (value table indexed by a byte permute, staged rows in the tables'
# second halves; padded rows without the sketch, swizzled rows with it), and
# the interleaved 4-bit pair and 2-bit quad tables.
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("kb,vb,qjl", [(3, 4, True), (3, 4, False), (4, 4, False), (2, 2, True)])
def test_gqa_groups(G, kb, vb, qjl):
    d, B, Hkv = 128, 1, 2
    lengths = [517]
    seed = G + 10 * kb + vb + 100 * qjl
    cb, cache, k, v, q = _setup(d, kb, vb, qjl, B, Hkv, G, lengths, 528, seed=seed, corr=True)
    out = tq.tq_decode_attention(cb, cache, q.cuda(), max_ctx=528)
    torch.cuda.synchronize()
    ref = _oracle(d, kb, vb, qjl, seed, k, v, q, lengths, G)
    assert_rows_close(out.cpu().numpy().reshape(-1, d), ref.reshape(-1, d))


def test_edge_lengths_and_empty():
    d, G, Hkv = 128, 4, 1
    lengths = [1, 127, 128, 129, 0, 255, 256, 16]
    B = len(lengths)
    cb, cache, k, v, q = _setup(d, 3, 4, False, B, Hkv, G, lengths, 256, seed=3, dtype=torch.float32)
    out = tq.tq_decode_attention(cb, cache, q.cuda(), max_ctx=256).cpu().numpy()
    ref = _oracle(d, 3, 4, False, 3, k, v, q, lengths, G)
    for b in range(B):
        if lengths[b] == 0:
            assert np.all(out[b] == 0)
        else:
            assert_rows_close(out[b], ref[b], what=f"len {lengths[b]}")


def test_softmax_scale_and_fp32_query():
    d, G, B, Hkv = 256, 2, 1, 3
    lengths = [200]
    cb, cache, k, v, q = _setup(d, 2, 3, True, B, Hkv, G, lengths, 208, seed=4, dtype=torch.float32)
    out = tq.tq_decode_attention(cb, cache, q.cuda(), softmax_scale=0.3, max_ctx=208)
    ref = _oracle(d, 2, 3, True, 4, k, v, q, lengths, G, scale=0.3)
    assert_rows_close(out.cpu().numpy().reshape(-1, d), ref.reshape(-1, d))


def test_deterministic_and_partition_independent():
    d, G, B, Hkv = 128, 2, 4, 8
    lengths = [3000, 2500, 1, 2999]
    cb, cache, k, v, q = _setup(d, 3, 4, True, B, Hkv, G, lengths, 8192, seed=8)
    qd = q.cuda()
    a = tq.tq_decode_attention(cb, cache, qd, max_ctx=3000)
    b = tq.tq_decode_attention(cb, cache, qd, max_ctx=3000)
    torch.cuda.synchronize()
    assert torch.equal(a, b)                                  # bit-identical reruns
    # the CTAs share out the tiles of all rows, so a longer row 2 moves every
    # later CTA boundary: rows 0, 1 and 3 are then merged from other partials
    cache.seq_lens[2] = 1700
    c = tq.tq_decode_attention(cb, cache, qd, max_ctx=3000)
    torch.cuda.synchronize()
    cache.seq_lens[2] = 1
    keep = [0, 1, 3]
    rel = ((a[keep] - c[keep]).abs().amax(-1) / a[keep].abs().amax(-1)).max().item()
    assert rel <= 1e-5
    assert not torch.equal(a[2], c[2])
    tb = oracle_tables(d, 3, 4, True, 8)
    for bb, h in ((0, 0), (3, 7), (2, 1)):
        n = lengths[bb]
        ek, ev = oracle_encode_unit(tb, k[bb, h, :n], v[bb, h, :n])
        ref = oracle_decode_unit(tb, q[bb, h * G:(h + 1) * G], ek, ev)
        assert_rows_close(a[bb, h * G:(h + 1) * G].cpu().numpy(), ref)
    ek, ev = oracle_encode_unit(tb, k[2, 5, :1700], v[2, 5, :1700])    # row 2 at its new length
    ref = oracle_decode_unit(tb, q[2, 5 * G:6 * G], ek, ev)
    assert_rows_close(c[2, 5 * G:6 * G].cpu().numpy(), ref)


def test_sphere_codebook_decode():
    d, G, B, Hkv = 128, 4, 2, 2
    lengths = [300, 129]
    g = torch.Generator().manual_seed(31)
    k = torch.randn(B, Hkv, 300, d, generator=g).bfloat16()
    v = torch.randn(B, Hkv, 300, d, generator=g).bfloat16()
    q = torch.randn(B, Hkv * G, d, generator=g).bfloat16()
    cb = tq.Codebook(d, 3, 4, True, seed=6, codebook="sphere")
    cache = tq.Cache(cb, B, Hkv, 304, "cuda")
    tq.tq_quantize_append(cb, cache, k.cuda(), v.cuda())
    cache.seq_lens.copy_(torch.tensor(lengths, dtype=torch.int32))
    out = tq.tq_decode_attention(cb, cache, q.cuda(), max_ctx=304).cpu()
    tb = oracle_tables(d, 3, 4, True, 6, codebook="sphere")
    for b in range(B):
        for h in range(Hkv):
            n = lengths[b]
            ek, ev = oracle_encode_unit(tb, k[b, h, :n], v[b, h, :n])
            ref = oracle_decode_unit(tb, q[b, h * G:(h + 1) * G], ek, ev)
            assert_rows_close(out[b, h * G:(h + 1) * G].numpy(), ref, what=f"({b},{h})")


def test_many_ragged_rows():
    # 300 rows (more than one 128-row chunk of the decode's schedule and one
    # 256-row pass of the combine's), a quarter of them empty, lengths 0..200:
    # most CTAs meet several units and some rows end inside a CTA's range
    d, G, B, Hkv = 128, 2, 300, 2
    rng = np.random.default_rng(11)
    lengths = [0 if rng.random() < 0.25 else int(rng.integers(1, 201)) for _ in range(B)]
    cb, cache, k, v, q = _setup(d, 3, 4, False, B, Hkv, G, lengths, 208, seed=12)
    out = tq.tq_decode_attention(cb, cache, q.cuda(), max_ctx=208).cpu()
    torch.cuda.synchronize()
    tb = oracle_tables(d, 3, 4, False, 12)
    for bb in list(range(0, B, 7)) + [B - 1]:
        for h in range(Hkv):
            n = lengths[bb]
            if n == 0:
                assert torch.all(out[bb, h * G:(h + 1) * G] == 0)
                continue
            ek, ev = oracle_encode_unit(tb, k[bb, h, :n], v[bb, h, :n])
            ref = oracle_decode_unit(tb, q[bb, h * G:(h + 1) * G], ek, ev)
            assert_rows_close(out[bb, h * G:(h + 1) * G].numpy(), ref, what=f"row {bb} head {h}")


def test_max_ctx_too_small_sets_flag():
    d, G, B, Hkv = 128, 1, 1, 1
    cb, cache, k, v, q = _setup(d, 3, 4, False, B, Hkv, G, [300], 512, seed=2)
    tq.tq_decode_attention(cb, cache, q.cuda(), max_ctx=128)
    torch.cuda.synchronize()
    assert int(cache.status.item()) & tq.TQ_FLAG_MAXCTX


def test_workspace_too_small_is_rejected():
    d = 128
    cb, cache, k, v, q = _setup(d, 3, 4, False, 1, 1, 1, [64], 64, seed=2)
    with pytest.raises(tq.TQError) as e:
        tq.tq_decode_attention(cb, cache, q.cuda(), max_ctx=64,
                               workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == tq.TQ_ERR_CAPACITY
