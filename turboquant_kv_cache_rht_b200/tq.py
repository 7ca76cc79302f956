"""Python binding of libtq (ctypes).  Argument marshalling only.

Every call below forwards to the C entry point of the same name in
``include/tq.h``; all codec and attention work runs in the CUDA kernels of
``libtq.so``.  PyTorch supplies device memory (the cache, inputs, outputs and
workspace are torch tensors owned by the caller) and the current CUDA stream.

Importing this module loads ``libtq.so`` from the package directory and raises
ImportError if it has not been built (``python -m
turboquant_kv_cache_rht_b200.build``); there is no fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import math
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtq.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libtq.so is not built ({_LIB_PATH}); run "
                      "`python -m turboquant_kv_cache_rht_b200.build`")
lib = C.CDLL(_LIB_PATH)

TQ_OK, TQ_ERR_INVALID, TQ_ERR_UNSUPPORTED, TQ_ERR_CUDA, TQ_ERR_CAPACITY, TQ_ERR_NOMEM = range(6)
TQ_FLAG_CAPACITY = 1
TQ_FLAG_MAXCTX = 2
TQ_FLAG_LAYOUT = 4
_DTYPES = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}
EXPORTS = ("tq_codebook_init", "tq_codebook_tables", "tq_quantize_append", "tq_quantize_cache",
           "tq_weights_quantize", "tq_lut_matmul_workspace_bytes", "tq_lut_matmul",
           "tq_decode_workspace_bytes", "tq_decode_attention", "tq_decode_attention_noalloc",
           "tq_free", "tq_last_error")


class tq_params(C.Structure):
    _fields_ = [("head_dim", C.c_int), ("k_bits", C.c_int), ("v_bits", C.c_int),
                ("qjl", C.c_int), ("seed", C.c_uint64), ("codebook", C.c_int)]


# TQ_CODEBOOK_GAUSSIAN, TQ_CODEBOOK_SPHERE, TQ_CODEBOOK_AFFINE
CODEBOOKS = {"gaussian": 0, "sphere": 1, "affine": 2}


class tq_layout(C.Structure):
    _fields_ = [("k_code_bytes", C.c_size_t), ("v_code_bytes", C.c_size_t),
                ("k_sign_bytes", C.c_size_t), ("norm_halves", C.c_size_t)]


class tq_cache(C.Structure):
    _fields_ = [("k_codes", C.c_void_p), ("v_codes", C.c_void_p), ("k_signs", C.c_void_p),
                ("k_norm", C.c_void_p), ("v_norm", C.c_void_p), ("k_rnorm", C.c_void_p),
                ("seq_lens", C.c_void_p), ("status", C.c_void_p), ("append_sync", C.c_void_p),
                ("batch", C.c_int), ("kv_heads", C.c_int), ("capacity", C.c_int)]


lib.tq_codebook_init.argtypes = [C.POINTER(tq_params), C.POINTER(C.c_void_p), C.POINTER(tq_layout)]
lib.tq_codebook_init.restype = C.c_int
lib.tq_codebook_tables.argtypes = [C.c_void_p] + [C.c_void_p] * 6
lib.tq_codebook_tables.restype = C.c_int
lib.tq_quantize_append.argtypes = [C.c_void_p, C.POINTER(tq_cache), C.c_void_p, C.c_void_p,
                                   C.c_int, C.c_int, C.c_void_p]
lib.tq_quantize_append.restype = C.c_int
lib.tq_quantize_cache.argtypes = [C.c_void_p, C.POINTER(tq_cache), C.c_void_p, C.c_void_p, C.c_int,
                                  C.c_int64, C.c_int64, C.c_int64, C.c_void_p, C.c_int, C.c_void_p]
lib.tq_quantize_cache.restype = C.c_int
lib.tq_weights_quantize.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_void_p,
                                    C.c_void_p, C.c_void_p]
lib.tq_weights_quantize.restype = C.c_int
lib.tq_lut_matmul_workspace_bytes.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_int]
lib.tq_lut_matmul_workspace_bytes.restype = C.c_size_t
lib.tq_lut_matmul.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_void_p,
                              C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]
lib.tq_lut_matmul.restype = C.c_int
lib.tq_decode_workspace_bytes.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int]
lib.tq_decode_workspace_bytes.restype = C.c_size_t
lib.tq_decode_attention.argtypes = [C.c_void_p, C.POINTER(tq_cache), C.c_void_p, C.c_int, C.c_int,
                                    C.c_float, C.c_int, C.c_void_p, C.c_void_p, C.c_size_t,
                                    C.c_void_p]
lib.tq_decode_attention.restype = C.c_int
lib.tq_decode_attention_noalloc.argtypes = [C.c_void_p, C.POINTER(tq_cache), C.c_void_p, C.c_int,
                                            C.c_int, C.c_float, C.c_int, C.c_void_p, C.c_void_p]
lib.tq_decode_attention_noalloc.restype = C.c_int
lib.tq_free.argtypes = [C.c_void_p]
lib.tq_free.restype = None
lib.tq_last_error.argtypes = []
lib.tq_last_error.restype = C.c_char_p


class TQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status}: {tq_last_error()}")


def tq_last_error() -> str:
    return lib.tq_last_error().decode()


def _check(st: int, where: str):
    if st != TQ_OK:
        raise TQError(st, where)


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def kv_bits_split(kv_bits: float) -> tuple[int, int]:
    """Key/value widths for a fractional kv_bits (3.5 -> 3-bit keys, 4-bit values)."""
    return int(math.floor(kv_bits + 1e-9)), int(math.ceil(kv_bits - 1e-9))


class Codebook:
    """Owner of a tq_codebook handle (host memory; freed with tq_free)."""

    def __init__(self, head_dim: int, k_bits: int, v_bits: int, qjl: bool = False, seed: int = 0,
                 codebook: str = "gaussian"):
        """codebook: "gaussian" (Lloyd-Max for N(0,1)), "sphere" (Lloyd-Max for
        the exact distribution of a rotated coordinate, which depends on head_dim)
        or "affine" (the affine group-64 comparison codec: rotated keys, fp16
        scale and bias per group of 64 channels)."""
        if codebook not in CODEBOOKS:
            raise ValueError(f"codebook must be one of {sorted(CODEBOOKS)}")
        self.params = tq_params(head_dim, k_bits, v_bits, int(bool(qjl)), seed & ((1 << 64) - 1),
                                CODEBOOKS[codebook])
        self.layout = tq_layout()
        h = C.c_void_p()
        _check(lib.tq_codebook_init(C.byref(self.params), C.byref(h), C.byref(self.layout)),
               "tq_codebook_init")
        self.handle = h

    @classmethod
    def from_kv_bits(cls, head_dim: int, kv_bits: float, qjl: bool = False, seed: int = 0,
                     codebook: str = "gaussian"):
        kb, vb = kv_bits_split(kv_bits)
        return cls(head_dim, kb, vb, qjl, seed, codebook)

    head_dim = property(lambda self: self.params.head_dim)
    k_bits = property(lambda self: self.params.k_bits)
    v_bits = property(lambda self: self.params.v_bits)
    qjl = property(lambda self: bool(self.params.qjl))
    affine = property(lambda self: self.params.codebook == CODEBOOKS["affine"])

    def tables(self) -> dict:
        """Host copies of the codebooks and rotation signs (tq_codebook_tables)."""
        lk, lv, d = 1 << self.k_bits, 1 << self.v_bits, self.head_dim
        kc, kb = (C.c_float * lk)(), (C.c_float * (lk - 1))()
        vc, vb = (C.c_float * lv)(), (C.c_float * (lv - 1))()
        s1, s2 = (C.c_int8 * d)(), (C.c_int8 * d)()
        _check(lib.tq_codebook_tables(self.handle, kc, kb, vc, vb, s1, s2), "tq_codebook_tables")
        to = lambda a, dt: torch.tensor(list(a), dtype=dt)
        return {"k_centroids": to(kc, torch.float32), "k_boundaries": to(kb, torch.float32),
                "v_centroids": to(vc, torch.float32), "v_boundaries": to(vb, torch.float32),
                "signs1": to(s1, torch.int8), "signs2": to(s2, torch.int8)}

    def __del__(self, _free=lib.tq_free):
        h = getattr(self, "handle", None)
        if h is not None and h.value:
            _free(h)
            self.handle = None


class Cache:
    """A compressed KV cache held in torch tensors (the caller owns them)."""

    def __init__(self, cb: Codebook, batch: int, kv_heads: int, capacity: int, device="cuda"):
        lay = cb.layout
        n = (batch, kv_heads, capacity)
        u8 = dict(dtype=torch.uint8, device=device)
        self.batch, self.kv_heads, self.capacity = batch, kv_heads, capacity
        self.k_codes = torch.zeros(*n, lay.k_code_bytes, **u8)
        self.v_codes = torch.zeros(*n, lay.v_code_bytes, **u8)
        self.k_signs = torch.zeros(*n, lay.k_sign_bytes, **u8) if cb.qjl else None
        # one fp16 norm per vector, or (scale, bias) per group for the affine codec
        nh = (lay.norm_halves,) if cb.affine else ()
        self.k_norm = torch.zeros(*n, *nh, dtype=torch.float16, device=device)
        self.v_norm = torch.zeros(*n, *nh, dtype=torch.float16, device=device)
        self.k_rnorm = torch.zeros(n, dtype=torch.float16, device=device) if cb.qjl else None
        self.seq_lens = torch.zeros(batch, dtype=torch.int32, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.append_sync = torch.zeros(batch, dtype=torch.int32, device=device)

    def struct(self) -> tq_cache:
        p = lambda t: None if t is None else t.data_ptr()
        return tq_cache(p(self.k_codes), p(self.v_codes), p(self.k_signs), p(self.k_norm),
                        p(self.v_norm), p(self.k_rnorm), p(self.seq_lens), p(self.status),
                        p(self.append_sync), self.batch, self.kv_heads, self.capacity)

    def nbytes(self) -> int:
        ts = [self.k_codes, self.v_codes, self.k_signs, self.k_norm, self.v_norm, self.k_rnorm]
        return sum(t.numel() * t.element_size() for t in ts if t is not None)


def _on_device(where: str, device: torch.device, **tensors) -> None:
    """The library takes device pointers: every tensor handed to it must be a
    CUDA tensor on the device of the cache (or of the encoded weights)."""
    for name, t in tensors.items():
        if t is not None and (not t.is_cuda or t.device != device):
            raise ValueError(f"{where}: {name} must be a CUDA tensor on {device}, not on {t.device}")


def _check_out(where: str, out: torch.Tensor, shape) -> None:
    if out.dtype != torch.float32 or tuple(out.shape) != tuple(shape) or not out.is_contiguous():
        raise ValueError(f"{where}: out must be a contiguous float32 tensor of shape {tuple(shape)}")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return _DTYPES[t.dtype]


def tq_quantize_append(cb: Codebook, cache: Cache, k: torch.Tensor, v: torch.Tensor,
                       stream=None) -> None:
    """k, v: [batch, kv_heads, n_new, head_dim] contiguous CUDA tensors of one dtype."""
    if k.shape != v.shape or k.dtype != v.dtype or k.dim() != 4:
        raise ValueError("k and v must be [batch, kv_heads, n_new, head_dim] of one dtype")
    if not (k.is_contiguous() and v.is_contiguous()):
        raise ValueError("k and v must be contiguous")
    if k.shape[0] != cache.batch or k.shape[1] != cache.kv_heads or k.shape[3] != cb.head_dim:
        raise ValueError(f"k shape {tuple(k.shape)} does not match the cache")
    _on_device("tq_quantize_append", cache.seq_lens.device, cache=cache.seq_lens, k=k, v=v)
    cs = cache.struct()
    _check(lib.tq_quantize_append(cb.handle, C.byref(cs), k.data_ptr(), v.data_ptr(),
                                  _dtype_code(k), k.shape[2], _stream_ptr(stream)),
           "tq_quantize_append")


def tq_quantize_cache(cb: Codebook, cache: Cache, k: torch.Tensor, v: torch.Tensor,
                      lengths: torch.Tensor | None = None, stream=None) -> None:
    """Convert a dense cache: k, v are [batch, kv_heads, T, head_dim] CUDA tensors
    of one dtype with unit channel stride and any other strides (a view of a
    [batch, T, kv_heads, head_dim] cache transposed works in place); lengths is
    an int32 CUDA tensor [batch] (default: T for every row).  Sets seq_lens."""
    if k.shape != v.shape or k.dtype != v.dtype or k.dim() != 4:
        raise ValueError("k and v must be [batch, kv_heads, T, head_dim] of one dtype")
    if k.stride() != v.stride() or k.stride(3) != 1:
        raise ValueError("k and v must share strides, with unit channel stride")
    if k.shape[0] != cache.batch or k.shape[1] != cache.kv_heads or k.shape[3] != cb.head_dim:
        raise ValueError(f"k shape {tuple(k.shape)} does not match the cache")
    T = k.shape[2]
    if lengths is None:
        lengths = torch.full((cache.batch,), T, dtype=torch.int32, device=k.device)
    if lengths.dtype != torch.int32 or lengths.shape != (cache.batch,) or not lengths.is_contiguous():
        raise ValueError("lengths must be a contiguous int32 tensor [batch]")
    _on_device("tq_quantize_cache", cache.seq_lens.device, cache=cache.seq_lens, k=k, v=v,
               lengths=lengths)
    cs = cache.struct()
    _check(lib.tq_quantize_cache(cb.handle, C.byref(cs), k.data_ptr(), v.data_ptr(), _dtype_code(k),
                                 k.stride(0), k.stride(1), k.stride(2), lengths.data_ptr(), T,
                                 _stream_ptr(stream)),
           "tq_quantize_cache")


def tq_lut_matmul_workspace_bytes(cb: Codebook, rows: int, k: int, m: int) -> int:
    return int(lib.tq_lut_matmul_workspace_bytes(cb.handle, rows, k, m))


class QuantizedWeights:
    """A weight matrix [rows, k] encoded block by block (blocks of head_dim input
    channels, the key codec): codes [k/d, rows, k_bits*d/8], fp16 norms [k/d, rows]."""

    def __init__(self, cb: Codebook, w: torch.Tensor, stream=None):
        if w.dim() != 2 or not w.is_contiguous():
            raise ValueError("w must be a contiguous [rows, k] CUDA tensor")
        _on_device("tq_weights_quantize", w.device, w=w)
        self.cb, (self.rows, self.k) = cb, w.shape
        nb = self.k // cb.head_dim
        self.codes = torch.empty(nb, self.rows, cb.layout.k_code_bytes, dtype=torch.uint8, device=w.device)
        self.norms = torch.empty(nb, self.rows, dtype=torch.float16, device=w.device)
        _check(lib.tq_weights_quantize(cb.handle, w.data_ptr(), _dtype_code(w), self.rows, self.k,
                                       self.codes.data_ptr(), self.norms.data_ptr(), _stream_ptr(stream)),
               "tq_weights_quantize")

    def copy(self) -> "QuantizedWeights":
        """A second copy of the encoded weights (new device buffers)."""
        c = QuantizedWeights.__new__(QuantizedWeights)
        c.cb, c.rows, c.k = self.cb, self.rows, self.k
        c.codes, c.norms = self.codes.clone(), self.norms.clone()
        return c

    def matmul(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        """x [m, k] CUDA tensor -> float32 [m, rows] = x W_hat^T."""
        if x.dim() != 2 or x.shape[1] != self.k or not x.is_contiguous():
            raise ValueError(f"x must be a contiguous [m, {self.k}] tensor")
        _on_device("tq_lut_matmul", self.codes.device, x=x)
        m = x.shape[0]
        y = torch.empty(m, self.rows, dtype=torch.float32, device=x.device)
        nbytes = tq_lut_matmul_workspace_bytes(self.cb, self.rows, self.k, m)
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
        _check(lib.tq_lut_matmul(self.cb.handle, self.codes.data_ptr(), self.norms.data_ptr(), self.rows,
                                 self.k, x.data_ptr(), _dtype_code(x), m, y.data_ptr(), ws.data_ptr(),
                                 nbytes, _stream_ptr(stream)),
               "tq_lut_matmul")
        return y


def tq_decode_workspace_bytes(cb: Codebook, batch: int, q_heads: int, kv_heads: int,
                              max_ctx: int) -> int:
    return int(lib.tq_decode_workspace_bytes(cb.handle, batch, q_heads, kv_heads, max_ctx))


def tq_decode_attention(cb: Codebook, cache: Cache, q: torch.Tensor, out: torch.Tensor | None = None,
                        softmax_scale: float = 0.0, max_ctx: int | None = None,
                        workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """q: [batch, q_heads, head_dim] CUDA tensor; returns float32 [batch, q_heads, head_dim]."""
    if q.dim() != 3 or q.shape[0] != cache.batch or q.shape[2] != cb.head_dim or not q.is_contiguous():
        raise ValueError("q must be contiguous [batch, q_heads, head_dim]")
    hq = q.shape[1]
    max_ctx = cache.capacity if max_ctx is None else max_ctx
    _on_device("tq_decode_attention", cache.seq_lens.device, cache=cache.seq_lens, q=q, out=out,
               workspace=workspace)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    _check_out("tq_decode_attention", out, q.shape)
    if workspace is None:   # (the library checks a caller's workspace size itself)
        need = tq_decode_workspace_bytes(cb, cache.batch, hq, cache.kv_heads, max_ctx)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    elif not workspace.is_contiguous():
        raise ValueError("tq_decode_attention: workspace must be contiguous")
    cs = cache.struct()
    _check(lib.tq_decode_attention(cb.handle, C.byref(cs), q.data_ptr(), _dtype_code(q), hq,
                                   float(softmax_scale), int(max_ctx), out.data_ptr(),
                                   workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                   _stream_ptr(stream)),
           "tq_decode_attention")
    return out


def tq_decode_attention_noalloc(cb: Codebook, cache: Cache, q: torch.Tensor,
                                out: torch.Tensor | None = None, softmax_scale: float = 0.0,
                                max_ctx: int | None = None, stream=None) -> torch.Tensor:
    """tq_decode_attention without a workspace, for callers that cannot
    allocate device memory: the library's built-in static scratch (8 MiB) is
    used instead.  Calls share that scratch, so they must not overlap on the
    GPU; make the first call on a device before any stream capture.  `out`
    should be passed by such callers (allocating it here is only a
    convenience)."""
    if q.dim() != 3 or q.shape[0] != cache.batch or q.shape[2] != cb.head_dim or not q.is_contiguous():
        raise ValueError("q must be contiguous [batch, q_heads, head_dim]")
    max_ctx = cache.capacity if max_ctx is None else max_ctx
    _on_device("tq_decode_attention_noalloc", cache.seq_lens.device, cache=cache.seq_lens, q=q,
               out=out)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    _check_out("tq_decode_attention_noalloc", out, q.shape)
    cs = cache.struct()
    _check(lib.tq_decode_attention_noalloc(cb.handle, C.byref(cs), q.data_ptr(), _dtype_code(q),
                                           q.shape[1], float(softmax_scale), int(max_ctx),
                                           out.data_ptr(), _stream_ptr(stream)),
           "tq_decode_attention_noalloc")
    return out


def tq_free(cb: Codebook) -> None:
    cb.__del__()
