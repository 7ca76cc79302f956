"""Host-side checks of the seeded input generators (CPU only)."""
import torch

from turboquant_kv_cache_rht_b200 import workloads as wl


def test_deterministic_and_sliceable():
    w = wl.with_sizes(wl.WORKLOADS["gqa"], context=64)
    k1, v1 = wl.kv_full(w)
    k2, v2 = wl.kv_unit(w, 0, 3, 64)
    assert k1.dtype == torch.bfloat16 and k1.shape == (1, 8, 64, 128)
    assert torch.equal(k1[0, 3], k2) and torch.equal(v1[0, 3], v2)
    assert not torch.equal(k1[0, 2], k1[0, 3])
    q1, q2 = wl.queries(w, 0), wl.queries(w, 0)
    assert torch.equal(q1, q2) and q1.shape == (1, 32, 128)
    assert not torch.equal(wl.queries(w, 1), q1)


def test_outlier_channels_fixed_over_tokens():
    w = wl.with_sizes(wl.WORKLOADS["gqa"], context=512)
    k, _ = wl.kv_unit(w, 0, 0, 512)
    rms = k.float().pow(2).mean(0).sqrt()
    assert int((rms > 5).sum()) == 4


def test_ragged_lengths_in_range():
    w = wl.WORKLOADS["serving"]
    lens = wl.context_lengths(w)
    assert len(lens) == 32 and all(8192 <= t <= 65536 for t in lens)
    assert len(set(lens)) > 20


def test_correlated_keys_have_cosine():
    w = wl.with_sizes(wl.WORKLOADS["qjl"], context=1000, batch=1)
    k, _ = wl.kv_unit(w, 0, 1, 1000)
    q = wl.queries(w, 0)[0].float()
    qn = q / q.norm(dim=-1, keepdim=True)
    kn = k.float() / k.float().norm(dim=-1, keepdim=True)
    cos = (kn @ qn[w.group:2 * w.group].T).max(dim=1).values
    assert int((cos > 0.78).sum()) == 10          # 1% of 1000 positions
    assert float(cos[cos > 0.78].min()) < 0.82
