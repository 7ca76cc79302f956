"""Host-side checks of the Python binding (CPU only: every call below is
rejected by the binding's own argument checks before the library is reached,
or touches host memory only)."""
import pytest
import torch

from turboquant_kv_cache_rht_b200 import tq


@pytest.mark.parametrize("codebook,nh", [("gaussian", None), ("sphere", None), ("affine", 4)])
def test_cache_arrays_follow_the_layout(codebook, nh):
    cb = tq.Codebook(128, 3, 4, qjl=True, codebook=codebook)
    c = tq.Cache(cb, 2, 3, 32, device="cpu")
    lay = cb.layout
    assert c.k_codes.shape == (2, 3, 32, lay.k_code_bytes) and c.v_codes.shape == (2, 3, 32, lay.v_code_bytes)
    assert c.k_signs.shape == (2, 3, 32, lay.k_sign_bytes) and c.k_rnorm.shape == (2, 3, 32)
    assert c.k_norm.shape == ((2, 3, 32) if nh is None else (2, 3, 32, nh)) == c.v_norm.shape
    per_vec = lay.k_code_bytes + lay.v_code_bytes + lay.k_sign_bytes + 2 + 2 * 2 * lay.norm_halves
    assert c.nbytes() == 2 * 3 * 32 * per_vec


def test_codebook_rejects_unknown_name():
    with pytest.raises(ValueError):
        tq.Codebook(128, 3, 4, codebook="uniform")


def test_append_and_decode_argument_checks():
    cb = tq.Codebook(128, 3, 4)
    c = tq.Cache(cb, 1, 2, 32, device="cpu")
    k = torch.zeros(1, 2, 4, 128)
    with pytest.raises(ValueError):
        tq.tq_quantize_append(cb, c, k, torch.zeros(1, 2, 5, 128))          # shapes differ
    with pytest.raises(ValueError):
        tq.tq_quantize_append(cb, c, k, k.half())                           # dtypes differ
    with pytest.raises(ValueError):
        tq.tq_quantize_append(cb, c, torch.zeros(1, 2, 4, 64), torch.zeros(1, 2, 4, 64))  # head_dim
    with pytest.raises(ValueError):
        kt = torch.zeros(1, 2, 128, 4).transpose(2, 3)
        tq.tq_quantize_append(cb, c, kt, kt)                                # not contiguous
    with pytest.raises(ValueError):
        tq.tq_quantize_cache(cb, c, k, k, lengths=torch.zeros(1, dtype=torch.int64))   # lengths dtype
    with pytest.raises(ValueError):
        tq.tq_decode_attention(cb, c, torch.zeros(1, 4, 64))                # q head_dim
    with pytest.raises(ValueError):
        tq.tq_decode_attention_noalloc(cb, c, torch.zeros(2, 4, 128))       # q batch


def test_weights_argument_checks():
    cb = tq.Codebook(128, 4, 4)
    with pytest.raises(ValueError):
        tq.QuantizedWeights(cb, torch.zeros(4, 16, 128))                    # not 2-D


def test_host_tensors_are_rejected_before_the_library():
    """The library takes device pointers; the binding refuses host tensors."""
    cb = tq.Codebook(128, 3, 4)
    c = tq.Cache(cb, 1, 2, 32, device="cpu")
    k = torch.zeros(1, 2, 4, 128)
    with pytest.raises(ValueError, match="CUDA tensor"):
        tq.tq_quantize_append(cb, c, k, k)
    with pytest.raises(ValueError, match="CUDA tensor"):
        tq.tq_quantize_cache(cb, c, k, k, lengths=torch.full((1,), 4, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA tensor"):
        tq.tq_decode_attention(cb, c, torch.zeros(1, 4, 128))
    with pytest.raises(ValueError, match="CUDA tensor"):
        tq.tq_decode_attention_noalloc(cb, c, torch.zeros(1, 4, 128))
    with pytest.raises(ValueError, match="CUDA tensor"):
        tq.QuantizedWeights(cb, torch.zeros(16, 128))


def test_output_buffer_checks():
    tq._check_out("decode", torch.zeros(2, 4, 128), (2, 4, 128))           # accepted
    for bad in (torch.zeros(2, 4, 64), torch.zeros(2, 4, 128, dtype=torch.float16),
                torch.zeros(2, 128, 4).transpose(1, 2)):
        with pytest.raises(ValueError, match="out must be"):
            tq._check_out("decode", bad, (2, 4, 128))
