"""GPU parity of the weights-regime LUT matmul vs the CPU oracle.

Weight codes and norms must equal the oracle's block encoding bit for bit, in
both lane layouts of the encoder.  Y = X W_hat^T must match the oracle's
float64 product within 2e-3 of each output row's largest magnitude.  Sizes
cover partial 64-row tiles, 1 to 9 inputs (partial 4-input tiles), plans with
and without a split of the blocks, and head_dim 64/128/256.  Repeated runs
are bit-identical, and the result tracks the unquantized X W^T within the
codec's distortion.
"""
import math

import numpy as np
import pytest
import torch

import oracle as o
from tests.tq_helpers import assert_rows_close

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("turboquant_kv_cache_rht_b200.tq")


def _setup(d, bits, rows, k, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(rows, k, generator=g)
    w[:, torch.randperm(k, generator=g)[:4]] *= 10.0
    w = w.to(dtype)
    cb = tq.Codebook(d, bits, bits, seed=seed)
    qw = tq.QuantizedWeights(cb, w.cuda())
    cent, bnd = o.codebook(bits)
    s1 = o.rotation_signs(seed, d)
    enc = o.weights_encode(w.float().numpy(), s1, cent, bnd, bits)
    return cb, qw, w, enc, cent, s1


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("rows", [48, 272])   # 48 x 4 blocks: one vector per warp; 272 x 16: 32 channels per lane
def test_weight_codes_bit_exact(d, bits, rows):
    k = 4 * d if rows == 48 else 16 * d
    cb, qw, w, enc, cent, s1 = _setup(d, bits, rows, k, seed=d + bits + rows)
    torch.cuda.synchronize()
    assert np.array_equal(qw.codes.cpu().numpy(), enc["codes"])
    assert np.array_equal(qw.norms.cpu().numpy().view(np.uint16), enc["norm16"].view(np.uint16))


@pytest.mark.parametrize("d,bits", [(128, 3), (128, 4), (64, 3), (64, 4), (256, 2), (256, 4)])
# m picks the column groups: 4 inputs per CTA up to 4, 8 up to 8, then 16
# (m = 9 and 16: one group of 16; m = 17: two, the second with one input)
@pytest.mark.parametrize("rows,k,m", [(80, 512, 1), (64, 1024, 3), (208, 256, 9), (4096, 4096, 1),
                                      (16, 2048, 5), (208, 512, 16), (80, 1024, 17)])
def test_matmul_matches_oracle(d, bits, rows, k, m):
    if k % d:
        pytest.skip("k is not a multiple of head_dim")
    cb, qw, w, enc, cent, s1 = _setup(d, bits, rows, k, seed=rows + k + m)
    x = torch.randn(m, k, generator=torch.Generator().manual_seed(m)).bfloat16()
    y = qw.matmul(x.cuda()).cpu().numpy()
    ref = o.lut_matmul(x.float().numpy(), enc["idx"], enc["norm16"], s1, cent)
    assert_rows_close(y, ref, what=f"rows {rows} k {k} m {m}")


def test_matmul_fp32_input_and_determinism():
    d, bits, rows, k, m = 128, 4, 96, 1024, 2
    cb, qw, w, enc, cent, s1 = _setup(d, bits, rows, k, seed=3, dtype=torch.float32)
    x = torch.randn(m, k, generator=torch.Generator().manual_seed(4))
    a = qw.matmul(x.cuda())
    b = qw.matmul(x.cuda())
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    ref = o.lut_matmul(x.numpy(), enc["idx"], enc["norm16"], s1, cent)
    assert_rows_close(a.cpu().numpy(), ref)
    assert tq.tq_lut_matmul_workspace_bytes(cb, rows, k, m) > 0      # this plan splits the blocks


def test_matmul_tracks_the_unquantized_product():
    d, bits, rows, k, m = 128, 4, 256, 2048, 4
    g = torch.Generator().manual_seed(12)
    w = torch.randn(rows, k, generator=g)
    x = torch.randn(m, k, generator=g)
    cb = tq.Codebook(d, bits, bits, seed=12)
    y = tq.QuantizedWeights(cb, w.cuda()).matmul(x.cuda()).cpu().double()
    exact = x.double() @ w.double().T
    rel = (torch.linalg.norm(y - exact) / torch.linalg.norm(exact)).item()
    assert rel < 1.3 * math.sqrt(0.009497)
