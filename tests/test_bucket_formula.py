"""The encode kernel's code search, restated on the host, against the definition.

The kernel does not count all 2^b - 1 boundaries.  It relies on the codebook's
odd symmetry (boundary L/2 - 1 is exactly 0, and boundary L/2 - 2 - q is the
negation of boundary L/2 + q) and searches only the positive ones:
    z > 0   ->  L/2 + #{p < |z|}
    z <= 0  ->  L/2 - 1 - #{p <= |z|},  with p <= a  taken as  p < nextup(a).
Here that formula is checked against the oracle's definition (#{boundaries
strictly below z}) at every boundary, at its float32 neighbours, at +-0, and on
random values.  The check runs in float32 with the same bit manipulation.
"""
import numpy as np
import pytest

import oracle as o


def _kernel_formula(z: np.ndarray, boundaries: np.ndarray) -> np.ndarray:
    levels = len(boundaries) + 1
    half = levels // 2
    p = boundaries[half:]                               # the positive boundaries, ascending
    z = z.astype(np.float32)
    pos = z > 0
    abits = z.view(np.uint32) & np.uint32(0x7FFFFFFF)
    key = (abits + np.where(pos, 0, 1).astype(np.uint32)).view(np.float32)
    cnt = (p[None, :] < key[:, None]).sum(axis=1)
    return np.where(pos, half + cnt, half - 1 - cnt)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_symmetric_search_equals_definition(bits):
    _, bnd = o.codebook(bits)
    assert bnd.dtype == np.float32
    half = (len(bnd) + 1) // 2
    assert bnd[half - 1] == 0.0 and np.array_equal(bnd[half:], -bnd[:half - 1][::-1])
    cands = [np.float32(0.0), np.float32(-0.0)]
    for b in bnd:
        for v in (b, -b):
            cands += [v, np.nextafter(v, np.float32(np.inf)), np.nextafter(v, np.float32(-np.inf))]
    cands += [np.float32(1e-45), np.float32(-1e-45), np.float32(11.3), np.float32(-11.3)]
    rng = np.random.default_rng(bits)
    cands += list(rng.standard_normal(20000).astype(np.float32) * 2)
    z = np.array(cands, dtype=np.float32)
    assert np.array_equal(_kernel_formula(z, bnd), o.bucket_index(z, bnd))
