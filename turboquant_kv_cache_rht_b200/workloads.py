"""Seeded synthetic inputs for the codec and the decode attention.

This module only draws numbers: it holds none of the codec's or the attention's
arithmetic, so both the CUDA path and the CPU oracle can take their inputs from
it.  Everything is generated on the CPU with ``torch.Generator`` (so a test can
regenerate any (batch row, KV head) slice on its own) and rounded to the
workload's storage dtype.

The shapes follow the TurboQuant pages' decode workloads: GQA models with
head_dim 128 or 256, long contexts, 2-4 bit codes (3.5 bits = 3-bit keys and
4-bit values), optional 1-bit QJL residual, and a ragged serving mix.  No public
dataset is used; keys and values are Gaussian with a few large outlier channels
per head (the case a random rotation is meant to spread out), and the QJL
workload plants keys correlated with the query (cosine 0.8) at 1% of positions.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    q_heads: int
    kv_heads: int
    head_dim: int
    k_bits: int
    v_bits: int
    qjl: bool
    dtype: str                      # "f32" | "bf16" | "f16" (K, V and q storage)
    seed: int
    rht_seed: int = 0
    context: int = 0                # fixed context length (0: ragged, see ctx_range)
    ctx_range: tuple = ()           # (lo, hi) inclusive, uniform per batch row
    outliers: int = 0               # outlier channels per KV head (fixed over tokens)
    outlier_scale: float = 1.0
    corr_frac: float = 0.0          # fraction of key positions correlated with the query
    corr_cos: float = 0.0
    codebook: str = "gaussian"      # "gaussian" | "sphere" | "affine" (the comparison codec)
    description: str = field(default="", compare=False)

    @property
    def group(self) -> int:
        return self.q_heads // self.kv_heads

    @property
    def torch_dtype(self):
        return {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[self.dtype]


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 1, 128, 4, 4, False, "f32", 1001, context=4096,
                     description="batch 1, 1 q / 1 KV head, d 128, ctx 4096, fp32 N(0,1), 4-bit K and V"),
    "gqa": Workload("gqa", 1, 32, 8, 128, 3, 4, False, "bf16", 1002, context=32768,
                    outliers=4, outlier_scale=20.0,
                    description="batch 1, 32 q / 8 KV heads, d 128, ctx 32768, bf16, 3-bit K + 4-bit V"),
    "qjl": Workload("qjl", 4, 32, 8, 128, 3, 4, True, "bf16", 1003, context=131072,
                    outliers=4, outlier_scale=20.0, corr_frac=0.01, corr_cos=0.8,
                    description="batch 4, 32 q / 8 KV heads, d 128, ctx 131072, bf16, "
                                "3-bit K + 1-bit QJL + 4-bit V, 1% keys at cosine 0.8 to the query"),
    "long": Workload("long", 1, 16, 4, 256, 2, 2, True, "bf16", 1004, context=524288,
                     outliers=4, outlier_scale=20.0,
                     description="batch 1, 16 q / 4 KV heads, d 256, ctx 524288, bf16, "
                                 "2-bit K + 1-bit QJL + 2-bit V"),
    "serving": Workload("serving", 32, 32, 8, 128, 3, 4, False, "bf16", 1005,
                        ctx_range=(8192, 65536), outliers=4, outlier_scale=20.0,
                        description="batch 32, 32 q / 8 KV heads, d 128, ragged ctx U[8k, 64k], "
                                    "bf16, 3-bit K + 4-bit V, 1 appended token per step"),
    "affine": Workload("affine", 1, 32, 8, 128, 4, 4, False, "bf16", 1006, context=32768,
                       outliers=4, outlier_scale=20.0, codebook="affine",
                       description="batch 1, 32 q / 8 KV heads, d 128, ctx 32768, bf16, affine "
                                   "group-64 comparison codec: rotated 4-bit K + 4-bit V"),
}


def derive_seed(base: int, *parts) -> int:
    """A 63-bit seed for one named slice of a workload."""
    h = hashlib.blake2b(repr((base,) + tuple(parts)).encode(), digest_size=8).digest()
    return int.from_bytes(h, "little") & ((1 << 63) - 1)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def context_lengths(w: Workload) -> list[int]:
    """Prefilled context length of every batch row."""
    if w.context:
        return [w.context] * w.batch
    lo, hi = w.ctx_range
    g = _gen(derive_seed(w.seed, "ctx"))
    return [int(t) for t in torch.randint(lo, hi + 1, (w.batch,), generator=g)]


def with_sizes(w: Workload, **changes) -> Workload:
    """Same recipe at other sizes (used for small parity cases)."""
    d = dict(w.__dict__)
    d.update(changes)
    return Workload(**d)


def queries(w: Workload, step: int = 0) -> torch.Tensor:
    """Decode queries [batch, q_heads, head_dim], N(0, 1), rounded to the storage dtype."""
    g = _gen(derive_seed(w.seed, "q", step))
    q = torch.randn(w.batch, w.q_heads, w.head_dim, generator=g)
    return q.to(w.torch_dtype)


def _outlier_channels(w: Workload, b: int, kvh: int, which: str) -> torch.Tensor:
    g = _gen(derive_seed(w.seed, "outliers", which, b, kvh))
    return torch.randperm(w.head_dim, generator=g)[: w.outliers]


def kv_unit(w: Workload, b: int, kvh: int, length: int, start: int = 0,
            step_tag=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Keys and values [length, head_dim] of one (batch row, KV head), storage dtype.

    ``start``/``step_tag`` name the slice: the prefill is (start 0, tag None);
    a token appended at decode step s uses tag ("step", s).  Outlier channels
    are the same for every slice of a unit.
    """
    d = w.head_dim
    tag = ("prefill",) if step_tag is None else tuple(step_tag) if isinstance(step_tag, tuple) else (step_tag,)
    gk = _gen(derive_seed(w.seed, "k", b, kvh, start, *tag))
    gv = _gen(derive_seed(w.seed, "v", b, kvh, start, *tag))
    k = torch.randn(length, d, generator=gk)
    v = torch.randn(length, d, generator=gv)
    if w.outliers:
        k[:, _outlier_channels(w, b, kvh, "k")] *= w.outlier_scale
        v[:, _outlier_channels(w, b, kvh, "v")] *= w.outlier_scale
    if w.corr_frac > 0 and step_tag is None and length > 0:
        k = _plant_correlated_keys(w, b, kvh, k)
    return k.to(w.torch_dtype), v.to(w.torch_dtype)


def _plant_correlated_keys(w: Workload, b: int, kvh: int, k: torch.Tensor) -> torch.Tensor:
    """Replace a random ``corr_frac`` of key rows by ||k|| (cos q_hat + sin e_perp).

    q_hat is the unit step-0 query of head h, cycling over the KV head's query
    heads in position order; e_perp is a random unit vector orthogonal to q_hat.
    """
    length, d = k.shape
    n_corr = max(1, int(round(w.corr_frac * length)))
    g = _gen(derive_seed(w.seed, "corr", b, kvh))
    pos = torch.sort(torch.randperm(length, generator=g)[:n_corr]).values
    q = queries(w, 0)[b].float()
    sin = (1.0 - w.corr_cos ** 2) ** 0.5
    e = torch.randn(n_corr, d, generator=g)
    k = k.clone()
    for j, t in enumerate(pos.tolist()):
        h = kvh * w.group + (j % w.group)
        qh = q[h] / q[h].norm()
        ep = e[j] - (e[j] @ qh) * qh
        ep = ep / ep.norm()
        k[t] = k[t].norm() * (w.corr_cos * qh + sin * ep)
    return k


def kv_full(w: Workload, lengths: list[int] | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """Prefill keys/values [batch, kv_heads, max_len, head_dim] (rows past a length are zero)."""
    lengths = context_lengths(w) if lengths is None else lengths
    tmax = max(lengths) if lengths else 0
    k = torch.zeros(w.batch, w.kv_heads, tmax, w.head_dim, dtype=w.torch_dtype)
    v = torch.zeros_like(k)
    for b in range(w.batch):
        for h in range(w.kv_heads):
            kk, vv = kv_unit(w, b, h, lengths[b])
            k[b, h, : lengths[b]] = kk
            v[b, h, : lengths[b]] = vv
    return k, v


def kv_step(w: Workload, step: int, n_new: int = 1) -> tuple[torch.Tensor, torch.Tensor]:
    """Keys/values appended at decode step ``step``: [batch, kv_heads, n_new, head_dim]."""
    k = torch.empty(w.batch, w.kv_heads, n_new, w.head_dim, dtype=w.torch_dtype)
    v = torch.empty_like(k)
    for b in range(w.batch):
        for h in range(w.kv_heads):
            kk, vv = kv_unit(w, b, h, n_new, step_tag=("step", step))
            k[b, h], v[b, h] = kk, vv
    return k, v
