"""Planted mistakes in the oracle must fail its pins (CPU only).

The oracle is trusted because its pins (closed forms, textbook tables, brute
force, a second route) are chosen so that a plausible mistake anywhere in it
fails one of them.  This file checks that claim directly.  Each case rewrites
one oracle function with one small, plausible mistake (a wrong shift, a
dropped factor, a flipped comparison, a transposed or misplaced operand),
swaps the mutant in for the duration of the case, and runs the pins of the
modules that guard that function until one fails.  A mutant that no pin
catches fails the case.  Nothing on disk changes; the mutant lives in a copy
of the oracle module's namespace, and monkeypatch puts the original back.
"""
from __future__ import annotations

import inspect
import itertools
import signal
import threading

import pytest

import oracle
import oracle.tq_oracle as tqo

import tests.test_oracle_affine as AFF
import tests.test_oracle_codebook as CB
import tests.test_oracle_codec as CODEC
import tests.test_oracle_decode as DEC
import tests.test_oracle_lut_matmul as LUT
import tests.test_oracle_rotation as ROT
import tests.test_oracle_sphere_codebook as SPH
from tests.conftest import read_golden

# (case id, oracle function, source fragment, its mutated form, pin modules)
MUTANTS = [
    # rotation: generator, signs, Hadamard matrix, transform, normalisation
    ("splitmix64-shift", "splitmix64", "(z >> 30)", "(z >> 31)", [ROT]),
    ("signs-from-low-bit", "rotation_signs", "(w >> 63)", "(w & 1)", [ROT]),
    ("second-rotation-seed", "rotation_signs", "(seed ^ GOLDEN64)", "(seed + 1)", [ROT, CODEC]),
    ("hadamard-or", "hadamard_matrix", "i[:, None] & i[None, :]", "i[:, None] | i[None, :]", [ROT]),
    ("fwht-butterfly-swapped", "fwht", "= a + b\n        w[..., 1, :] = a - b",
     "= a - b\n        w[..., 1, :] = a + b", [ROT]),
    ("fwht-last-stage-dropped", "fwht", "while h < d:", "while 2 * h < d:", [ROT]),
    ("rht-unnormalised", "rht_forward", " / math.sqrt(x.shape[-1])", "", [ROT]),
    ("rht-inverse-order", "rht_inverse", "signs * fwht(y, np.float64)", "fwht(signs * y, np.float64)",
     [ROT]),
    ("pairwise-sum-sequential", "pairwise_sum_f32", "x = x[..., 0::2] + x[..., 1::2]",
     "x = np.concatenate([x[..., :1] + x[..., 1:2], x[..., 2:]], axis=-1)", [ROT]),
    # Lloyd-Max codebooks
    ("gaussian-tail-scale", "_upper_tail", "x / _SQRT2", "x / 2.0", [CB]),
    ("codebook-mirror-index", "codebook", "c64[half - 1 - j]", "c64[half - j]", [CB]),
    ("codebook-boundaries-not-midpoints", "codebook", "(cent[:-1] + cent[1:]) * np.float32(0.5)",
     "cent[:-1]", [CB, CODEC]),
    ("sphere-density-exponent", "sphere_density", "((d - 3) / 2)", "((d - 2) / 2)", [SPH]),
    ("sphere-moment-factor", "sphere_first_moment", "c * d / (d - 1) * (g(a) - g(b))",
     "c * (g(a) - g(b))", [SPH]),
    ("sphere-beta-parameter", "_sphere_upper_tail", "betaincc(0.5, (d - 1) / 2,",
     "betaincc(0.5, d / 2,", [SPH]),
    ("sphere-mirror-index", "sphere_codebook", "c64[half - 1 - j]", "c64[half - j]", [SPH]),
    # codec
    ("bucket-ties-up", "bucket_index", "(b < z)", "(b <= z)", [CODEC]),
    ("pack-big-endian", "pack_codes", 'bitorder="little"', 'bitorder="big"', [CODEC]),
    ("pack-msb-first", "pack_codes", ">> np.arange(bits))", ">> np.arange(bits)[::-1])", [CODEC]),
    ("unpack-big-endian", "unpack_codes", 'bitorder="little"', 'bitorder="big"', [CODEC]),
    ("encode-multiplies-by-norm", "encode", "z = u * inv[:, None]", "z = u * n[:, None]", [CODEC]),
    ("norm-not-square-rooted", "encode", "n = np.sqrt(pairwise_sum_f32(x * x))",
     "n = pairwise_sum_f32(x * x)", [CODEC]),
    ("no-sign-flips", "encode", "u = fwht(np.where(s1 < 0, -x, x))", "u = fwht(x)", [CODEC]),
    ("qjl-residual-without-norm", "encode", "r = u - n16.astype(np.float32)[:, None] * centroids[idx]",
     "r = u - centroids[idx]", [CODEC]),
    ("qjl-rho-unscaled", "encode", "rho = np.sqrt(pairwise_sum_f32(r * r)) / np.sqrt(np.float32(d))",
     "rho = np.sqrt(pairwise_sum_f32(r * r))", [CODEC]),
    ("qjl-sign-of-zero", "encode", "sbits = (w >= 0)", "sbits = (w > 0)", [CODEC]),
    ("qjl-reuses-first-rotation", "encode", "w = fwht(np.where(s2 < 0, -r, r))",
     "w = fwht(np.where(s1 < 0, -r, r))", [CODEC]),
    # decode attention
    ("decode-scale-dropped", "decode_attention", "scores = scale * scores", "scores = scores", [DEC]),
    ("decode-qjl-constant", "decode_attention", "math.sqrt(math.pi / (2 * d))",
     "math.sqrt(2 / (math.pi * d))", [DEC]),
    ("decode-qjl-sign-map", "decode_attention", "sgn = 2.0 * np.asarray(k_sign_bits, np.float64) - 1.0",
     "sgn = np.asarray(k_sign_bits, np.float64)", [DEC]),
    ("decode-softmax-over-all-rows", "decode_attention", "/ p.sum(axis=-1, keepdims=True)",
     "/ p.sum()", [DEC]),
    ("decode-no-inverse-rotation", "decode_attention", "return rht_inverse(o_rot, s1)", "return o_rot",
     [DEC]),
    ("decode-query-not-rotated", "decode_attention", "q_rot = rht_forward(q, s1)", "q_rot = q", [DEC]),
    ("dequantize-unscaled", "dequantize_rotated", " / math.sqrt(d))", ")", [DEC]),
    ("dense-unscaled", "dense_attention", "default_scale(q.shape[-1], sm_scale) * ", "", [DEC]),
    ("default-scale-1-over-d", "default_scale", "1.0 / math.sqrt(d)", "1.0 / d", [DEC]),
    ("second-route-qjl-transposed", "decode_attention_dequant_route", "(q @ r1.T @ r2.T)",
     "(q @ r1 @ r2.T)", [DEC]),
    ("kv-bits-swapped", "kv_bits_split", "int(math.floor(kv_bits + 1e-9)), int(math.ceil(kv_bits - 1e-9))",
     "int(math.ceil(kv_bits - 1e-9)), int(math.floor(kv_bits + 1e-9))", [DEC]),
    # weights regime
    ("weights-strided-blocks", "weights_encode", "w.reshape(n, k // d, d).transpose(1, 0, 2)",
     "w.reshape(n, d, k // d).transpose(2, 0, 1)", [LUT]),
    ("weights-left-rotated", "weights_dequantize",
     "rht_inverse(dequantize_rotated(idx[j], norm16[j], centroids), s1)",
     "dequantize_rotated(idx[j], norm16[j], centroids)", [LUT]),
    # affine comparison codec
    ("affine-bias-is-max", "affine_encode", "bias16 = mn.astype(np.float16)",
     "bias16 = mx.astype(np.float16)", [AFF]),
    ("affine-levels", "affine_encode", "levels = np.float32((1 << bits) - 1)",
     "levels = np.float32(1 << bits)", [AFF]),
    ("affine-floor", "affine_encode", "t = np.rint((yg - bf) / sf)", "t = np.floor((yg - bf) / sf)", [AFF]),
    ("affine-strided-groups", "affine_encode", "yg = y.reshape(n, ng, AFFINE_GROUP)",
     "yg = y.reshape(n, AFFINE_GROUP, ng).transpose(0, 2, 1)", [AFF]),
    ("affine-rotation-unnormalised", "affine_encode", "y = fwht(np.where(s1 < 0, -x, x)) * rs",
     "y = fwht(np.where(s1 < 0, -x, x))", [AFF]),
    ("affine-residual-sign", "affine_encode", "\n        r = y - y_hat\n", "\n        r = y_hat - y\n",
     [AFF]),
    ("affine-bytes-without-signs", "affine_vector_bytes", "((d // 8 + 2) if qjl else 0)",
     "(2 if qjl else 0)", [AFF]),
    ("affine-bias-subtracted", "affine_dequantize", "(s * idx.reshape(n, ng, AFFINE_GROUP) + b)",
     "(s * idx.reshape(n, ng, AFFINE_GROUP) - b)", [AFF]),
    ("affine-query-not-rotated", "affine_decode_attention",
     "q_rot = rht_forward(q, s1) if s1 is not None else q", "q_rot = q", [AFF]),
]


def _mutant(name: str, old: str, new: str):
    src = inspect.getsource(getattr(tqo, name))
    assert src.count(old) == 1, f"{name}: the fragment must occur exactly once"
    ns = dict(vars(tqo))
    exec(compile(src.replace(old, new), f"<mutant of {name}>", "exec"), ns)
    return ns[name]


def _pins(module):
    """Every test function of ``module`` with every parameter combination of
    its parametrize marks, in definition order."""
    for name, fn in vars(module).items():
        if not (name.startswith("test_") and inspect.isfunction(fn)):
            continue
        axes = []
        for mark in getattr(fn, "pytestmark", []):
            if mark.name == "parametrize":
                names, values = mark.args[0], mark.args[1]
                names = [s.strip() for s in names.split(",")] if isinstance(names, str) else list(names)
                axes.append([dict(zip(names, v if len(names) > 1 else (v,))) for v in values])
        for combo in itertools.product(*axes):
            kw = {k: v for part in combo for k, v in part.items()}
            if "golden" in inspect.signature(fn).parameters:
                kw["golden"] = read_golden
            yield f"{module.__name__.split('.')[-1]}::{name}{kw if kw else ''}", fn, kw


class _TooSlow(Exception):
    pass


def _caught(fn, kw, seconds=30) -> bool:
    """True when the pin fails (an assertion, an error, or no answer within
    ``seconds``: an iteration that stops converging counts as caught; the
    limit needs SIGALRM and the main thread, and is skipped without them)."""
    timed = hasattr(signal, "SIGALRM") and threading.current_thread() is threading.main_thread()

    def alarm(*_):
        raise _TooSlow()
    if timed:
        old = signal.signal(signal.SIGALRM, alarm)
        signal.alarm(seconds)
    try:
        fn(**kw)
        return False
    except Exception:
        return True
    finally:
        if timed:
            signal.alarm(0)
            signal.signal(signal.SIGALRM, old)


@pytest.mark.parametrize("case,name,old,new,modules", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(monkeypatch, case, name, old, new, modules):
    mutant = _mutant(name, old, new)
    monkeypatch.setattr(tqo, name, mutant)
    if hasattr(oracle, name):
        monkeypatch.setattr(oracle, name, mutant)
    for pin_id, fn, kw in (p for m in modules for p in _pins(m)):
        if _caught(fn, kw):
            return
    pytest.fail(f"no pin in {[m.__name__ for m in modules]} catches the mutant {case}")


def test_unmutated_oracle_passes_the_same_pins():
    """The harness itself: with no mutant every collected pin passes."""
    seen = set()
    for m in (ROT, CB, CODEC, DEC, SPH, LUT, AFF):
        for pin_id, fn, kw in _pins(m):
            assert not _caught(fn, kw), pin_id
            seen.add(pin_id.split("::")[0])
    assert len(seen) == 7
