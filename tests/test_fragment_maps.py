"""Host-side check of the decode kernel's channel-to-MMA-slot maps (CPU only).

The decode kernel assigns channels to the k-slots of its m16n8k16 score MMAs
and to the rows of its value MMAs freely (the reduction order is free), in a
way that lets every thread read one contiguous slice of a packed row.  These
maps are restated here from their definitions and checked for what the
kernel relies on:

* keys, Lloyd-Max codec: thread quarter q, k-block kb: slots (2q, 2q+1) carry
  channels (c0, c0+1) and slots (2q+8, 2q+9) carry (c0+2, c0+3), with
  c0 = q*d/4 + 4*kb -- every channel exactly once, and the pair's bit offset
  inside the quarter's slice is b*4*kb;
* keys, affine codec: c0 = 64*(kb/4) + 16*q + 4*(kb%4) -- every channel once,
  every k-block inside one 64-channel group, the bit offset inside the
  quarter's slice of that group b*4*(kb%4);
* QJL signs: d >= 128, slots (2q, 2q+1) are bits (j, j+16) and (2q+8, 2q+9)
  bits (j+8, j+24) of word kb/8 of the quarter (j = kb%8); d = 64, the
  quarter's 16 bits h with its copy shifted by 8 give (h[kb], h[kb+8]) and
  (h[kb+4], h[kb+12]) -- every channel once, matching the query columns;
* values: thread group g, m-block mb: row g is channel g*d/8 + 2*mb and row
  g+8 channel g*d/8 + 2*mb + 1 -- every channel once, and a thread's value
  channels lie in one 64-channel group (one (scale, bias) pair per token).
"""
import pytest

DIMS = [64, 128, 256]


def _key_slots(d, affine):
    """(q, kb, slot) -> channel of the score MMA's k dimension."""
    m = {}
    for q in range(4):
        for kb in range(d // 16):
            c0 = 64 * (kb >> 2) + 16 * q + 4 * (kb & 3) if affine else q * (d // 4) + 4 * kb
            for slot, ch in zip((2 * q, 2 * q + 1, 2 * q + 8, 2 * q + 9), (c0, c0 + 1, c0 + 2, c0 + 3)):
                m[(q, kb, slot)] = ch
    return m


@pytest.mark.parametrize("d", DIMS)
@pytest.mark.parametrize("affine", [False, True])
def test_key_slots_cover_every_channel_once(d, affine):
    m = _key_slots(d, affine)
    assert sorted(m.values()) == list(range(d))
    for kb in range(d // 16):                    # the 16 slots of one k-block are distinct
        assert sorted(s for (q, k, s) in m if k == kb) == list(range(16))


@pytest.mark.parametrize("d", DIMS)
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_key_pairs_sit_where_the_slice_reads_them(d, bits):
    """The code pair of slots (2q, 2q+1) starts at bit b*4*kb of quarter q's
    slice (Lloyd-Max) or at b*4*(kb%4) of its slice of group kb/4 (affine)."""
    for affine in (False, True):
        m = _key_slots(d, affine)
        for q in range(4):
            for kb in range(d // 16):
                c0 = m[(q, kb, 2 * q)]
                if affine:
                    slice_start = 64 * (kb >> 2) + 16 * q
                    assert bits * (c0 - slice_start) == bits * 4 * (kb & 3)
                    assert 0 <= c0 - slice_start and c0 + 3 - slice_start < 16
                else:
                    slice_start = q * (d // 4)
                    assert bits * (c0 - slice_start) == bits * 4 * kb
                    assert c0 + 3 - slice_start < d // 4


@pytest.mark.parametrize("d", DIMS)
def test_affine_k_blocks_lie_in_one_group(d):
    m = _key_slots(d, True)
    for kb in range(d // 16):
        groups = {ch // 64 for (q, k, s), ch in m.items() if k == kb}
        assert groups == {kb >> 2}


def _sign_channels(d, q, kb):
    """Channels of the four sign slots (2q, 2q+1, 2q+8, 2q+9), read off the
    bit positions the kernel shifts to bits 15 and 31."""
    if d >= 128:
        word, j = kb >> 3, kb & 7
        base = q * (d // 4) + 32 * word
        return base + j, base + j + 16, base + j + 8, base + j + 24
    # x = h | (h << 8), h the quarter's 16 bits.  (x << (15 - kb)) brings x's bits
    # kb and kb + 16 to 15 and 31; (x << (11 - kb)) bits kb + 4 and kb + 20.  Only
    # bits 0-7 (h itself) and 16-23 (the shifted copy) are read, never the
    # overlap 8-15.
    pos = (kb, kb + 16, kb + 4, kb + 20)
    assert all(p < 8 or 16 <= p < 24 for p in pos)
    h_of = lambda p: p if p < 8 else p - 8
    return tuple(q * 16 + h_of(p) for p in (kb, kb + 16, kb + 4, kb + 20))


@pytest.mark.parametrize("d", DIMS)
def test_sign_slots_match_query_columns(d):
    """The query columns take r2[base], r2[base + P1], r2[base + P2], r2[base + P3]."""
    chans = []
    for q in range(4):
        for kb in range(d // 16):
            got = _sign_channels(d, q, kb)
            if d >= 128:
                base = q * (d // 4) + 32 * (kb >> 3) + (kb & 7)
                p1, p2, p3 = 16, 8, 24
            else:
                base = q * 16 + kb
                p1, p2, p3 = 8, 4, 12
            assert got == (base, base + p1, base + p2, base + p3)
            chans.extend(got)
    assert sorted(chans) == list(range(d))


@pytest.mark.parametrize("d", DIMS)
def test_value_rows_cover_every_channel_once_within_one_group(d):
    chans = []
    for g in range(8):
        own = []
        for mb in range(d // 16):
            own += [g * (d // 8) + 2 * mb, g * (d // 8) + 2 * mb + 1]     # rows g, g + 8
        assert own == list(range(g * (d // 8), (g + 1) * (d // 8)))
        assert {c // 64 for c in own} == {(g * (d // 8)) // 64}           # one affine group
        chans += own
    assert sorted(chans) == list(range(d))
