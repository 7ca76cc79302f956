"""Host-side check of the decode's work partition, restated from its definition.

The token tiles of all (batch row, KV head) units are laid end to end (unit
(b, h) covers tiles [H*P_b + h*n_b, H*P_b + (h+1)*n_b), P_b the tiles of the
rows before b), CTA c of N takes tiles [floor(c*T/N), floor((c+1)*T/N)), each
(CTA, unit) segment writes its partial to slot c + u, and the merge of unit u
reads the CTAs c_lo..c_hi given by closed forms.  These properties are what the
kernels rely on; here they are checked exhaustively on random shapes:
every tile belongs to exactly one segment, slots are distinct and below
N + U - 1, and the closed-form CTA range of every unit is exactly the set of
CTAs whose range meets it (plus empty CTAs, which the merge skips).
"""
import numpy as np
import pytest

TILE = 64


def _units(lengths, heads):
    n = [(L + TILE - 1) // TILE for L in lengths]
    starts, p = [], 0
    for b, nb in enumerate(n):
        for h in range(heads):
            starts.append((heads * p + h * nb, nb))
        p += nb
    return starts, heads * p


def _cta_range(c, total, ctas):
    return c * total // ctas, (c + 1) * total // ctas


@pytest.mark.parametrize("seed", range(40))
def test_partition_properties(seed):
    rng = np.random.default_rng(seed)
    batch = int(rng.integers(1, 40))
    heads = int(rng.choice([1, 2, 4, 8]))
    lengths = [int(x) if rng.random() > 0.2 else 0 for x in rng.integers(0, 3000, batch)]
    units, total = _units(lengths, heads)
    ctas = int(rng.integers(1, 600))
    owner = {}
    slots = set()
    for c in range(ctas):
        t0, t1 = _cta_range(c, total, ctas)
        for u, (us, n) in enumerate(units):
            lo, hi = max(t0, us), min(t1, us + n)
            if lo >= hi:
                continue
            slot = c + u
            assert slot not in slots and slot <= (ctas - 1) + (len(units) - 1)
            slots.add(slot)
            for t in range(lo, hi):
                assert t not in owner
                owner[t] = c
    assert sorted(owner) == list(range(total))          # every tile exactly once
    if total == 0:
        return
    for u, (su, n) in enumerate(units):
        if n == 0:
            continue
        eu = su + n
        c_lo = ((su + 1) * ctas + total - 1) // total - 1
        c_hi = (eu * ctas + total - 1) // total - 1
        meets = {c for c in range(ctas) if max(_cta_range(c, total, ctas)[0], su) < min(_cta_range(c, total, ctas)[1], eu)}
        assert meets and min(meets) == c_lo and max(meets) == c_hi
        for c in range(c_lo, c_hi + 1):                 # the gaps are CTAs with empty ranges
            if c not in meets:
                a, b = _cta_range(c, total, ctas)
                assert a == b
