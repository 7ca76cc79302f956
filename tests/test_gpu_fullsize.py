"""Full-size parity on sampled outputs (GPU).

Each workload is built at its full size (context 32k / 131k / 524k / ragged
8k-64k), one step is taken exactly as bench.py takes it (append one token per
(batch row, KV head), then decode with the max_ctx and therefore the split plan
bench.py uses), and the outputs of a few (batch row, KV head) units -- all of
their query heads -- are compared with the oracle, which encodes the same
seeded keys and values itself.  Codes of the sampled units are also compared
bit for bit.  The oracle is computed unit by unit, so these run in seconds to
a minute each on the host.
"""
import numpy as np
import pytest
import torch

import bench
from tests.tq_helpers import assert_rows_close, oracle_decode_unit, oracle_encode_unit, oracle_tables
from turboquant_kv_cache_rht_b200 import workloads as wl

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("turboquant_kv_cache_rht_b200.tq")

CASES = {
    "gqa": [(0, 0), (0, 7), (0, 3)],
    "qjl": [(0, 0), (3, 7), (2, 4)],
    "long": [(0, 0), (0, 3)],
    "serving": [(0, 0), (31, 7), (17, 2)],
    "tiny": [(0, 0)],
    "affine": [(0, 0), (0, 7), (0, 2)],
}


def _run_step(w, dev):
    plan = bench.replica_plan(w, bench.default_steps_total(), torch.cuda.get_device_properties(dev).L2_cache_size)
    lengths, cap, max_ctx = plan["lengths"], plan["capacity"], plan["max_ctx"]
    cb = tq.Codebook(w.head_dim, w.k_bits, w.v_bits, w.qjl, w.rht_seed, codebook=w.codebook)
    cache = tq.Cache(cb, w.batch, w.kv_heads, cap, dev)
    tmax = max(lengths)
    for h in range(w.kv_heads):          # bulk prefill, one KV head at a time (as bench.py)
        kh = torch.zeros(w.batch, 1, tmax, w.head_dim, dtype=w.torch_dtype)
        vh = torch.zeros_like(kh)
        for b in range(w.batch):
            k, v = wl.kv_unit(w, b, h, lengths[b])
            kh[b, 0, :lengths[b]] = k
            vh[b, 0, :lengths[b]] = v
        tmp = tq.Cache(cb, w.batch, 1, cap, dev)
        tq.tq_quantize_append(cb, tmp, kh.to(dev), vh.to(dev))
        for name in ("k_codes", "v_codes", "k_signs", "k_norm", "v_norm", "k_rnorm"):
            src = getattr(tmp, name)
            if src is not None:
                getattr(cache, name)[:, h].copy_(src[:, 0])
        del tmp, kh, vh
    cache.seq_lens.copy_(torch.tensor(lengths, dtype=torch.int32))
    k_new, v_new = wl.kv_step(w, 0)
    tq.tq_quantize_append(cb, cache, k_new.to(dev).contiguous(), v_new.to(dev).contiguous())
    q = wl.queries(w, 0)
    out = tq.tq_decode_attention(cb, cache, q.to(dev), max_ctx=max_ctx)
    torch.cuda.synchronize(dev)
    assert int(cache.status.item()) == 0
    assert cache.seq_lens.cpu().tolist() == [L + 1 for L in lengths]
    return cache, out.cpu(), lengths, k_new, v_new, q


@pytest.mark.parametrize("name", list(CASES))
def test_full_size_sampled_units(name):
    w = wl.WORKLOADS[name]
    dev = torch.device("cuda", 0)
    cache, out, lengths, k_new, v_new, q = _run_step(w, dev)
    tb = oracle_tables(w.head_dim, w.k_bits, w.v_bits, w.qjl, w.rht_seed, codebook=w.codebook)
    G = w.group
    for b, h in CASES[name]:
        k, v = wl.kv_unit(w, b, h, lengths[b])
        k_all = torch.cat([k, k_new[b, h]])
        v_all = torch.cat([v, v_new[b, h]])
        ek, ev = oracle_encode_unit(tb, k_all, v_all)
        n = lengths[b] + 1
        assert np.array_equal(cache.k_codes[b, h, :n].cpu().numpy(), ek["codes"])
        assert np.array_equal(cache.v_codes[b, h, :n].cpu().numpy(), ev["codes"])
        ref = oracle_decode_unit(tb, q[b, h * G:(h + 1) * G], ek, ev)
        assert_rows_close(out[b, h * G:(h + 1) * G].numpy(), ref, what=f"{name} unit ({b},{h})")
