"""Shared helpers of the GPU parity tests: run the CUDA path, run the oracle on
the same seeded inputs, compare.  Oracle inputs come from the seeded generators
only, never from the CUDA path."""
from __future__ import annotations

import numpy as np
import torch

import oracle as o

DEC_TOL = 2e-3   # decode: per row, max |gpu - oracle| <= DEC_TOL * max |oracle|


def oracle_tables(head_dim, k_bits, v_bits, qjl, seed, codebook="gaussian"):
    if codebook == "affine":      # the affine group-64 comparison codec: signs only
        s2 = o.rotation_signs(seed, head_dim, second=True) if qjl else None
        return dict(affine=True, s1=o.rotation_signs(seed, head_dim), s2=s2, k_bits=k_bits,
                    v_bits=v_bits)
    book = (lambda b: o.codebook(b)) if codebook == "gaussian" else (lambda b: o.sphere_codebook(b, head_dim))
    ck, bk = book(k_bits)
    cv, bv = book(v_bits)
    s1 = o.rotation_signs(seed, head_dim)
    s2 = o.rotation_signs(seed, head_dim, second=True) if qjl else None
    return dict(ck=ck, bk=bk, cv=cv, bv=bv, s1=s1, s2=s2, k_bits=k_bits, v_bits=v_bits)


def oracle_encode_unit(tb, k, v):
    """Oracle encoding of one (batch row, KV head): k, v torch [T, d] (any float dtype)."""
    kf = k.float().numpy()
    vf = v.float().numpy()
    if tb.get("affine"):          # keys rotated, values as they are
        return (o.affine_encode(kf, tb["k_bits"], tb["s1"], tb["s2"]),
                o.affine_encode(vf, tb["v_bits"]))
    ek = o.encode(kf, tb["s1"], tb["ck"], tb["bk"], tb["k_bits"], tb["s2"])
    ev = o.encode(vf, tb["s1"], tb["cv"], tb["bv"], tb["v_bits"])
    return ek, ev


def oracle_decode_unit(tb, q_rows, ek, ev, scale=None):
    if tb.get("affine"):
        return o.affine_decode_attention(q_rows.float().numpy().astype(np.float64), tb["s1"], ek, ev,
                                         sm_scale=scale, s2=tb["s2"])
    kw = {}
    if tb["s2"] is not None:
        kw = dict(s2=tb["s2"], k_sign_bits=ek["sign_bits"], k_rnorm16=ek["rnorm16"])
    return o.decode_attention(q_rows.float().numpy().astype(np.float64), tb["s1"], ek["idx"],
                              ek["norm16"], tb["ck"], ev["idx"], ev["norm16"], tb["cv"],
                              sm_scale=scale, **kw)


def assert_rows_close(gpu, ref, tol=DEC_TOL, what=""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape
    for r in range(ref.shape[0]):
        scale = np.abs(ref[r]).max()
        err = np.abs(gpu[r] - ref[r]).max()
        assert err <= tol * scale + 1e-30, f"{what} row {r}: max err {err:.3e} vs {tol} * {scale:.3e}"


def cache_slot_bytes(t: torch.Tensor, b, h, lo, hi):
    return t[b, h, lo:hi].cpu().numpy()


def half_bits(t: torch.Tensor, b, h, lo, hi):
    return t[b, h, lo:hi].cpu().view(torch.int16).numpy().view(np.uint16)
