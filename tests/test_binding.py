"""Host-side checks of the Python binding (CPU only: every call below is
rejected by the binding's own argument checks before the library is reached,
or touches host memory only)."""
import os
import re

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


def test_missing_library_fails_loudly(tmp_path):
    """Without libtq.so next to it the binding refuses to import: there is no
    fallback implementation to drop back to."""
    import importlib.util
    import shutil
    src = os.path.join(os.path.dirname(os.path.abspath(tq.__file__)), "tq.py")
    shutil.copy(src, tmp_path / "tq.py")
    spec = importlib.util.spec_from_file_location("tq_without_library", tmp_path / "tq.py")
    with pytest.raises(ImportError, match="libtq.so is not built"):
        spec.loader.exec_module(importlib.util.module_from_spec(spec))


def test_product_never_imports_the_oracle():
    """The oracle is test infrastructure: no product source names it."""
    pkg = os.path.dirname(os.path.abspath(tq.__file__))
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "tq_oracle" not in text, f
