"""C-ABI checks that need no GPU: exports, host-side tables, argument validation."""
import ctypes as C
import os
import re

import numpy as np
import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle as o
from turboquant_kv_cache_rht_b200 import tq

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "tq.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z_0-9]+)\s*\(", src)))


def test_plain_c_client(tmp_path):
    """include/tq.h compiles as strict C99 and as C++17, and a program linked
    against libtq.so gets the same answers as the Python binding (host-only
    calls)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.dirname(os.path.abspath(tq.__file__))
    src = os.path.join(root, "tests", "native", "abi_from_c.c")
    outputs = []
    # as C99, and the same source as C++ (the header's extern "C" linkage)
    for lang, std in (("c", "-std=c99"), ("c++", "-std=c++17")):
        exe = tmp_path / f"abi_from_{lang.replace('+', 'p')}"
        build = subprocess.run([cc, "-x", lang, std, "-pedantic", "-Wall", "-Wextra", "-Werror",
                                "-I", os.path.join(root, "include"), src, "-x", "none",
                                "-L", pkg, "-ltq", f"-Wl,-rpath,{pkg}", "-o", str(exe)]
                               + (["-lstdc++"] if lang == "c++" else []),
                               capture_output=True, text=True, timeout=120)
        assert build.returncode == 0, build.stderr
        run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
        assert run.returncode == 0, run.stdout + run.stderr
        outputs.append(run.stdout)
    assert outputs[0] == outputs[1]
    got = {ln.split()[0]: ln.split()[1:] for ln in outputs[0].splitlines() if ln.strip()}
    cb = tq.Codebook(128, 3, 4, qjl=True, seed=42)
    t = cb.tables()
    assert got["init"] == ["0"] and got["tables"] == ["0"]
    lay = cb.layout
    assert got["layout"] == [str(x) for x in (lay.k_code_bytes, lay.v_code_bytes, lay.k_sign_bytes,
                                              lay.norm_halves)]
    assert np.array_equal(np.array(got["k_centroids"], np.float32), t["k_centroids"].numpy())
    assert [int(x) for x in got["signs1"]] == t["signs1"].tolist()[:16]
    assert int(got["decode_ws"][0]) == tq.tq_decode_workspace_bytes(cb, 32, 32, 8, 65536)
    assert int(got["lut_ws"][0]) == tq.tq_lut_matmul_workspace_bytes(cb, 16384, 8192, 16)
    assert got["rejected"][0] == str(tq.TQ_ERR_INVALID) and "cache is NULL" in " ".join(got["rejected"])


def test_last_error_is_per_thread():
    """Each thread reads the message of its own last failing call."""
    import threading
    cb = tq.Codebook(128, 3, 4)
    barrier = threading.Barrier(2)
    seen = {}

    def worker(name, fail):
        for _ in range(200):
            fail()
            barrier.wait()          # the other thread has failed differently in between
            seen.setdefault(name, set()).add(tq.tq_last_error())
            barrier.wait()

    fails = {"capacity": lambda: _append(cb, _fake_cache(capacity=40)),
             "dtype": lambda: _append(cb, _fake_cache(), dtype=7)}
    threads = [threading.Thread(target=worker, args=(n, f)) for n, f in fails.items()]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=60)
    assert len(seen["capacity"]) == 1 and "multiple of 16" in next(iter(seen["capacity"]))
    assert len(seen["dtype"]) == 1 and "unknown dtype" in next(iter(seen["dtype"]))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert set(names) == set(tq.EXPORTS)
    for n in names:
        assert hasattr(tq.lib, n), n


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kb,vb", [(2, 2), (3, 4), (4, 4), (2, 3)])
@pytest.mark.parametrize("seed", [0, 1234567, 2**64 - 1])
def test_tables_equal_oracle_bit_for_bit(d, kb, vb, seed):
    cb = tq.Codebook(d, kb, vb, qjl=True, seed=seed)
    t = cb.tables()
    for bits, c_name, b_name in ((kb, "k_centroids", "k_boundaries"), (vb, "v_centroids", "v_boundaries")):
        cent, bnd = o.codebook(bits)
        assert np.array_equal(t[c_name].numpy().view(np.uint32), cent.view(np.uint32))
        assert np.array_equal(t[b_name].numpy().view(np.uint32), bnd.view(np.uint32))
    assert np.array_equal(t["signs1"].numpy(), o.rotation_signs(seed, d))
    assert np.array_equal(t["signs2"].numpy(), o.rotation_signs(seed, d, second=True))


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kb,vb", [(2, 2), (3, 4), (4, 4), (2, 3), (3, 3)])
def test_sphere_tables_equal_oracle_bit_for_bit(d, kb, vb):
    """The host solves the sphere codebook with its own integration (Gauss-Legendre
    cell masses), the oracle with the incomplete beta function; the float32 tables
    must agree bit for bit."""
    cb = tq.Codebook(d, kb, vb, codebook="sphere")
    t = cb.tables()
    for bits, c_name, b_name in ((kb, "k_centroids", "k_boundaries"), (vb, "v_centroids", "v_boundaries")):
        cent, bnd = o.sphere_codebook(bits, d)
        assert np.array_equal(t[c_name].numpy().view(np.uint32), cent.view(np.uint32))
        assert np.array_equal(t[b_name].numpy().view(np.uint32), bnd.view(np.uint32))
    assert not np.array_equal(t["k_centroids"].numpy(), o.codebook(kb)[0])   # differs from N(0,1)


def test_layout_bytes():
    cb = tq.Codebook(128, 3, 4, qjl=True)
    assert (cb.layout.k_code_bytes, cb.layout.v_code_bytes, cb.layout.k_sign_bytes) == (48, 64, 16)
    cb = tq.Codebook(256, 2, 2, qjl=False)
    assert (cb.layout.k_code_bytes, cb.layout.v_code_bytes, cb.layout.k_sign_bytes) == (64, 64, 0)


@pytest.mark.parametrize("bad", [dict(head_dim=96), dict(head_dim=512), dict(k_bits=1),
                                 dict(v_bits=5), dict(qjl=2), dict(codebook=3), dict(codebook=-1)])
def test_codebook_rejects_bad_params(bad):
    p = dict(head_dim=128, k_bits=3, v_bits=4, qjl=0, seed=0, codebook=0)
    p.update(bad)
    params = tq.tq_params(p["head_dim"], p["k_bits"], p["v_bits"], p["qjl"], p["seed"], p["codebook"])
    h = C.c_void_p()
    assert tq.lib.tq_codebook_init(C.byref(params), C.byref(h), None) == tq.TQ_ERR_INVALID
    assert not h.value
    assert tq.tq_last_error()


def test_codebook_init_null_arguments():
    params = tq.tq_params(128, 3, 4, 0, 0, 0)
    h = C.c_void_p()
    assert tq.lib.tq_codebook_init(None, C.byref(h), None) == tq.TQ_ERR_INVALID
    assert tq.lib.tq_codebook_init(C.byref(params), None, None) == tq.TQ_ERR_INVALID
    # a NULL layout is allowed; any table buffer may be NULL; tq_free(NULL) is a no-op
    assert tq.lib.tq_codebook_init(C.byref(params), C.byref(h), None) == tq.TQ_OK and h.value
    assert tq.lib.tq_codebook_tables(h, None, None, None, None, None, None) == tq.TQ_OK
    kc = (C.c_float * 8)()
    assert tq.lib.tq_codebook_tables(h, kc, None, None, None, None, None) == tq.TQ_OK
    assert list(kc) == tq.Codebook(128, 3, 4).tables()["k_centroids"].tolist()
    tq.lib.tq_free(h)
    tq.lib.tq_free(None)


def test_affine_layout_matches_the_pages_memory_table(golden):
    """The library's per-vector bytes for the affine codec reproduce the
    "Memory footprint over long context" KB/token figures (the fp16 row fixes
    the cached channels per token; head_dim 128)."""
    rows = {r[0]: (int(r[1]), int(r[2]), int(r[3]), float(r[4])) for r in golden("kv_memory_footprint.txt")}
    vectors = rows["fp16"][3] * 1024 / (2 * 2) / 128
    for name in ("affine4", "turboquant4", "turboquant3_qjl"):
        kb, vb, qjl, want = rows[name]
        lay = tq.Codebook(128, kb, vb, qjl=bool(qjl), codebook="affine").layout
        per_vec = (lay.k_code_bytes + lay.v_code_bytes + lay.k_sign_bytes + (2 if qjl else 0)
                   + 2 * (2 * lay.norm_halves))                     # fp16 metadata of K and V
        assert abs(per_vec * vectors / 1024 - want) <= 0.05, name
    assert tq.Codebook(128, 4, 4).layout.norm_halves == 1
    assert tq.Codebook(256, 2, 3, codebook="affine").layout.norm_halves == 8


def test_affine_tables_are_integer_levels():
    t = tq.Codebook(64, 3, 4, codebook="affine").tables()
    assert t["k_centroids"].tolist() == list(range(8)) and t["v_centroids"].tolist() == list(range(16))
    assert t["k_boundaries"].tolist() == [j + 0.5 for j in range(7)]


def test_head_dim_64_layout():
    cb = tq.Codebook(64, 3, 4, qjl=True)
    assert (cb.layout.k_code_bytes, cb.layout.v_code_bytes, cb.layout.k_sign_bytes) == (24, 32, 8)
    assert tq.Codebook(64, 3, 4, codebook="sphere").tables()["k_centroids"].shape[0] == 8


def _fake_cache(batch=2, kv_heads=2, capacity=64, qjl=False, **over):
    """A tq_cache struct with aligned fake addresses: validation reads no memory."""
    a = iter(range(1 << 20, 1 << 30, 1 << 16))
    c = tq.tq_cache(next(a), next(a), next(a) if qjl else None, next(a), next(a),
                    next(a) if qjl else None, next(a), next(a), next(a), batch, kv_heads, capacity)
    for k, v in over.items():
        setattr(c, k, v)
    return c


def _append(cb, cache, n_new=1, k=1 << 12, v=1 << 13, dtype=1):
    return tq.lib.tq_quantize_append(cb.handle, C.byref(cache), k, v, dtype, n_new, None)


def test_append_validation():
    cb = tq.Codebook(128, 3, 4)
    assert _append(cb, _fake_cache(capacity=40)) == tq.TQ_ERR_INVALID      # not a multiple of 16
    assert "multiple of 16" in tq.tq_last_error()
    assert _append(cb, _fake_cache(k_codes=None)) == tq.TQ_ERR_INVALID
    assert _append(cb, _fake_cache(k_norm=(1 << 20) + 2)) == tq.TQ_ERR_INVALID   # misaligned
    assert _append(cb, _fake_cache(batch=0)) == tq.TQ_ERR_INVALID
    assert _append(cb, _fake_cache(), n_new=-1) == tq.TQ_ERR_INVALID
    assert _append(cb, _fake_cache(), dtype=7) == tq.TQ_ERR_INVALID
    assert _append(cb, _fake_cache(), k=0) == tq.TQ_ERR_INVALID
    assert _append(cb, _fake_cache(), k=(1 << 12) + 4) == tq.TQ_ERR_INVALID
    assert _append(cb, _fake_cache(), n_new=0) == tq.TQ_OK                 # no-op, no launch
    assert _append(cb, _fake_cache(), n_new=65) == tq.TQ_ERR_INVALID       # past the capacity
    assert "exceeds capacity" in tq.tq_last_error()
    assert _append(cb, _fake_cache(batch=65536)) == tq.TQ_ERR_INVALID      # one grid row per batch row
    assert "65535" in tq.tq_last_error()
    big = dict(batch=65535, kv_heads=1 << 30, capacity=1 << 30)             # sizes only
    assert _append(cb, _fake_cache(**big)) == tq.TQ_ERR_INVALID
    assert "too large" in tq.tq_last_error()
    qcb = tq.Codebook(128, 3, 4, qjl=True)
    assert _append(qcb, _fake_cache()) == tq.TQ_ERR_INVALID                # QJL needs k_signs
    assert _append(qcb, _fake_cache(qjl=True, k_rnorm=(1 << 21) + 2)) == tq.TQ_ERR_INVALID
    assert "not 16-byte aligned" in tq.tq_last_error()
    assert tq.lib.tq_quantize_append(None, C.byref(_fake_cache()), 1 << 12, 1 << 13, 1, 1,
                                     None) == tq.TQ_ERR_INVALID


def _convert(cb, cache, k=1 << 12, v=1 << 13, dtype=1, strides=(2 * 64 * 128, 64 * 128, 128),
             lengths=1 << 14, max_len=64):
    return tq.lib.tq_quantize_cache(cb.handle, C.byref(cache), k, v, dtype, *strides, lengths,
                                    max_len, None)


def test_convert_validation():
    """Rejected before any launch (the pointers are fake; no GPU is touched)."""
    cb = tq.Codebook(128, 3, 4)
    assert _convert(cb, _fake_cache(capacity=40)) == tq.TQ_ERR_INVALID        # capacity % 16
    assert _convert(cb, _fake_cache(), dtype=7) == tq.TQ_ERR_INVALID
    assert _convert(cb, _fake_cache(), max_len=-1) == tq.TQ_ERR_INVALID
    assert _convert(cb, _fake_cache(), max_len=0) == tq.TQ_OK                 # no-op, no launch
    assert _convert(cb, _fake_cache(), k=0) == tq.TQ_ERR_INVALID
    assert _convert(cb, _fake_cache(), lengths=0) == tq.TQ_ERR_INVALID
    assert _convert(cb, _fake_cache(), lengths=(1 << 14) + 2) == tq.TQ_ERR_INVALID   # misaligned
    assert _convert(cb, _fake_cache(), k=(1 << 12) + 8) == tq.TQ_ERR_INVALID         # misaligned
    assert _convert(cb, _fake_cache(), strides=(1, 128, 128)) == tq.TQ_ERR_INVALID   # 2 bytes
    assert _convert(cb, _fake_cache(), strides=(64, 128, 4)) == tq.TQ_ERR_INVALID    # 8 bytes
    assert _convert(cb, _fake_cache(), strides=(-128, 128, 128)) == tq.TQ_ERR_INVALID


def test_weights_validation():
    """Rejected before any launch (fake pointers; no GPU is touched)."""
    cb = tq.Codebook(128, 4, 4)
    wq = lambda rows=64, k=512, dtype=1, w=1 << 12, codes=1 << 13, norms=1 << 14: tq.lib.tq_weights_quantize(
        cb.handle, w, dtype, rows, k, codes, norms, None)
    assert wq(rows=40) == tq.TQ_ERR_INVALID          # not a multiple of 16
    assert wq(k=500) == tq.TQ_ERR_INVALID            # not a multiple of head_dim
    assert wq(dtype=9) == tq.TQ_ERR_INVALID
    assert wq(w=0) == tq.TQ_ERR_INVALID
    assert wq(codes=(1 << 13) + 4) == tq.TQ_ERR_INVALID
    acb = tq.Codebook(128, 4, 4, codebook="affine")                # weights take Lloyd-Max codes
    assert tq.lib.tq_weights_quantize(acb.handle, 1 << 12, 1, 64, 512, 1 << 13, 1 << 14,
                                      None) == tq.TQ_ERR_UNSUPPORTED
    mm = lambda rows=64, k=512, m=1, ws=0, nbytes=0, y=1 << 15: tq.lib.tq_lut_matmul(
        cb.handle, 1 << 13, 1 << 14, rows, k, 1 << 12, 1, m, y, ws, nbytes, None)
    assert mm(m=0) == tq.TQ_ERR_INVALID
    assert mm(m=65535 * 4 + 1) == tq.TQ_ERR_INVALID
    assert mm(y=0) == tq.TQ_ERR_INVALID
    assert mm(y=(1 << 15) + 8) == tq.TQ_ERR_INVALID   # misaligned output
    need = tq.tq_lut_matmul_workspace_bytes(cb, 64, 512, 1)
    assert need > 0 and mm(ws=1 << 16, nbytes=need - 4) == tq.TQ_ERR_CAPACITY
    assert mm(ws=(1 << 16) + 4, nbytes=need) == tq.TQ_ERR_INVALID       # misaligned workspace
    assert tq.tq_lut_matmul_workspace_bytes(cb, 64, 500, 1) == 0       # bad k
    # rotated inputs: 4 blocks x 1 group of 4 inputs x (8 k-blocks x 32 lanes x 2 words
    # + 4 scales); 64 rows x 1 group is one tile, so the 4 blocks are split one per
    # CTA and the partial sums (4 x 1 x 64) follow
    assert need == (4 * 1 * 8 * 32 * 2 + 4 * 1 * 4 + 4 * 1 * 64) * 4
    # more 128-row tiles than the 592-CTA bound need no split: rotated inputs only
    # (8 inputs -> one group of 8)
    assert tq.tq_lut_matmul_workspace_bytes(cb, 128 * 600, 512, 8) == (4 * 2 * 8 * 64 + 4 * 8) * 4


def _decode(cb, cache, q_heads=4, max_ctx=64, ws=1 << 14, ws_bytes=1 << 30, scale=0.0, q=1 << 12,
            out=1 << 13):
    return tq.lib.tq_decode_attention(cb.handle, C.byref(cache), q, 1, q_heads, scale, max_ctx,
                                      out, ws, ws_bytes, None)


def test_decode_validation():
    cb = tq.Codebook(128, 3, 4)
    assert _decode(cb, _fake_cache(), q_heads=3) == tq.TQ_ERR_INVALID       # not a multiple
    assert _decode(cb, _fake_cache(), max_ctx=65) == tq.TQ_ERR_INVALID      # past capacity
    assert _decode(cb, _fake_cache(), ws_bytes=16) == tq.TQ_ERR_CAPACITY
    assert _decode(cb, _fake_cache(), q=0) == tq.TQ_ERR_INVALID
    assert _decode(cb, _fake_cache(), max_ctx=-1) == tq.TQ_ERR_INVALID
    assert _decode(cb, _fake_cache(batch=70000)) == tq.TQ_ERR_INVALID       # merge grid rows
    assert _decode(cb, _fake_cache(), q=(1 << 12) + 2) == tq.TQ_ERR_INVALID     # misaligned q
    assert _decode(cb, _fake_cache(), out=(1 << 13) + 4) == tq.TQ_ERR_INVALID   # misaligned out
    assert _decode(cb, _fake_cache(), ws=(1 << 14) + 8) == tq.TQ_ERR_INVALID    # misaligned workspace
    assert "16-byte aligned" in tq.tq_last_error()
    assert _decode(cb, _fake_cache(), ws=0) == tq.TQ_ERR_CAPACITY              # no workspace
    assert _decode(cb, _fake_cache(), scale=float("nan")) == tq.TQ_ERR_INVALID
    assert _decode(cb, _fake_cache(kv_heads=1), q_heads=3) == tq.TQ_ERR_UNSUPPORTED   # group 3
    assert _decode(cb, _fake_cache(kv_heads=1), q_heads=16) == tq.TQ_ERR_UNSUPPORTED  # group 16
    cb35 = tq.Codebook(128, 4, 2)
    assert _decode(cb35, _fake_cache()) == tq.TQ_ERR_UNSUPPORTED           # v_bits < k_bits


def test_workspace_size_formula():
    # slots (one wave of at most 592 CTAs, no more CTAs than tiles, + units - 1)
    # x group x (head_dim + 2) floats
    def expect(batch, q_heads, kv_heads, max_ctx, d=128):
        return _expect_decode_workspace(batch, q_heads, kv_heads, max_ctx, d)
    cb = tq.Codebook(128, 3, 4)
    for args in ((1, 32, 8, 32768), (32, 32, 8, 65536), (1, 1, 1, 100), (1, 1, 1, 0), (4, 8, 8, 64)):
        assert tq.tq_decode_workspace_bytes(cb, *args) == expect(*args), args
    assert tq.tq_decode_workspace_bytes(cb, 1, 30, 8, 100) == 0              # group 3.75
    cb256 = tq.Codebook(256, 2, 2)
    assert tq.tq_decode_workspace_bytes(cb256, 2, 16, 4, 524288) == expect(2, 16, 4, 524288, 256)


def _expect_decode_workspace(batch, q_heads, kv_heads, max_ctx, d):
    units = batch * kv_heads
    ctas = max(1, min(148 * 4, units * max(1, -(-max_ctx // 64))))
    return (ctas + units - 1) * (q_heads // kv_heads) * (d + 2) * 4


@settings(max_examples=300, deadline=None)
@given(batch=st.integers(1, 300), kv_heads=st.sampled_from([1, 2, 4, 8, 16]),
       group=st.sampled_from([1, 2, 4, 8]), max_ctx=st.integers(0, 1 << 21),
       d=st.sampled_from([64, 128, 256]))
def test_decode_workspace_formula_random(batch, kv_heads, group, max_ctx, d):
    cb = _codebook_cache(d)
    got = tq.tq_decode_workspace_bytes(cb, batch, kv_heads * group, kv_heads, max_ctx)
    assert got == _expect_decode_workspace(batch, kv_heads * group, kv_heads, max_ctx, d)


def _expect_lut_workspace(rows, k, m, d, max_ctas=148 * 4):
    """The weights-regime plan restated: 128-row tiles times column groups of
    4, 8 or 16 inputs; the k/d blocks split so that tiles x splits stays within
    one wave; workspace = rotated inputs + their scales + split partials."""
    per_group = 16 if m > 8 else 8 if m > 4 else 4
    groups = -(-m // per_group)
    tiles = max(1, -(-rows // 128) * groups)
    nblocks = max(1, k // d)
    s = max(1, min(nblocks, max_ctas // tiles))
    per_split = -(-nblocks // s)
    splits = -(-nblocks // per_split)
    frag_words = nblocks * groups * (per_group // 4) * (d // 16) * 64
    scales = nblocks * groups * per_group
    partials = splits * m * rows if splits > 1 else 0
    return (frag_words + scales + partials) * 4


@settings(max_examples=300, deadline=None)
@given(rows=st.integers(1, 2048).map(lambda r: 16 * r), blocks=st.integers(1, 96),
       m=st.integers(1, 64), d=st.sampled_from([64, 128, 256]))
def test_lut_workspace_formula_random(rows, blocks, m, d):
    cb = _codebook_cache(d)
    assert tq.tq_lut_matmul_workspace_bytes(cb, rows, blocks * d, m) == _expect_lut_workspace(
        rows, blocks * d, m, d)


_CODEBOOKS = {}


def _codebook_cache(d):
    if d not in _CODEBOOKS:
        _CODEBOOKS[d] = tq.Codebook(d, 4, 4)
    return _CODEBOOKS[d]


def test_kv_bits_split_matches_oracle():
    for b in (2, 2.5, 3, 3.5, 4):
        assert tq.kv_bits_split(b) == o.kv_bits_split(b)


@pytest.mark.parametrize("name", ["tiny", "gqa", "qjl", "long", "serving", "affine"])
def test_bench_byte_model_matches_the_layout(name):
    """bench.py's algorithmic bytes per stored (token, KV head) equal what the
    library's layout says a decode must read: codes, the fp16 norm or (scale,
    bias) words of K and V, and with QJL the sign plane plus an fp16 norm."""
    import bench
    from turboquant_kv_cache_rht_b200 import workloads as wl
    w = wl.WORKLOADS[name]
    lay = tq.Codebook(w.head_dim, w.k_bits, w.v_bits, w.qjl, codebook=w.codebook).layout
    per_token = (lay.k_code_bytes + lay.v_code_bytes + 2 * 2 * lay.norm_halves
                 + ((lay.k_sign_bytes + 2) if w.qjl else 0))
    assert bench.token_bytes(w) == per_token
    # and the arrays a cache allocates from that layout hold exactly that much
    cb = tq.Codebook(w.head_dim, w.k_bits, w.v_bits, w.qjl, codebook=w.codebook)
    assert tq.Cache(cb, 2, 3, 32, device="cpu").nbytes() == 2 * 3 * 32 * per_token


def test_bench_step_bytes():
    """3.5 bits at d 128 reads 48 + 64 + 4 bytes per (token, KV head), 4.41x
    fewer than bf16; a step's decode bytes are the rows' cache bytes plus the
    bf16 queries read and fp32 outputs written, its append one K and one V
    vector in and out per (row, KV head)."""
    import bench
    from turboquant_kv_cache_rht_b200 import workloads as wl
    assert bench.token_bytes(wl.WORKLOADS["serving"]) == 116
    w = wl.with_sizes(wl.WORKLOADS["gqa"], context=100, batch=3)
    lens = [100, 37, 0]
    sb = bench.step_bytes(w, lens)
    d = w.head_dim
    assert sb["decode"] == sum(lens) * w.kv_heads * 116 + w.batch * w.q_heads * d * (2 + 4)
    assert sb["append"] == w.batch * w.kv_heads * (2 * d * 2 + (3 + 4) * d // 8 + 4)
    assert sb["total"] == sb["decode"] + sb["append"]
