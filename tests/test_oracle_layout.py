"""Pins of the oracle's page layout: bijection, hand-derived addresses, round trip,
byte accounting, and that the layout feeds the sm_80+ ``mma.sync`` A-operand
fragments through the nibble extraction the decode kernel performs."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_addresses_are_a_bijection():
    for g in (8, 16):
        for side in ("K", "V"):
            tb = oracle.tokens_per_block(g)
            seen = {oracle.block_bit_address(g, side, t, k) for t in range(tb) for k in range(g)}
            assert len(seen) == 256
            assert all(0 <= w < 8 and 0 <= b < 32 for w, b in seen)


def test_hand_derived_addresses():
    with open(os.path.join(GOLDEN, "layout_bits.txt")) as f:
        rows = [l.split("|") for l in f if l.strip() and not l.startswith("#")]
    assert rows
    for r in rows:
        g, side, tau, k, word, bit = int(r[0]), r[1].strip(), int(r[2]), int(r[3]), int(r[4]), int(r[5])
        assert oracle.block_bit_address(g, side, tau, k) == (word, bit), r


@pytest.mark.parametrize("g", [8, 16])
@pytest.mark.parametrize("b", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("side", ["K", "V"])
def test_round_trip(g, b, side):
    rng = np.random.default_rng(g * 100 + b * 10 + (side == "V"))
    P = 64
    plane_off, sz_off = 16, 16 + b * P * g // 8
    page = rng.integers(0, 256, size=sz_off + 4 * P + 16, dtype=np.uint8)
    tokens = np.array([0, 1, 5, 17, 31, 32, 63])
    codes = rng.integers(0, 2 ** b, size=(len(tokens), g)).astype(np.uint8)
    s = rng.standard_normal(len(tokens)).astype(np.float16)
    z = rng.standard_normal(len(tokens)).astype(np.float16)
    before = page.copy()
    oracle.pack_group_into_page(page, g, side, P, b, plane_off, sz_off, tokens, codes, s, z)
    c2, s2, z2 = oracle.unpack_group_from_page(page, g, side, P, b, plane_off, sz_off, P)
    np.testing.assert_array_equal(c2[tokens], codes)
    np.testing.assert_array_equal(s2[tokens], s)
    np.testing.assert_array_equal(z2[tokens], z)
    # other tokens keep their bits
    c0, s0, z0 = oracle.unpack_group_from_page(before, g, side, P, b, plane_off, sz_off, P)
    other = np.setdiff1d(np.arange(P), tokens)
    np.testing.assert_array_equal(c2[other], c0[other])
    np.testing.assert_array_equal(s2[other].view(np.uint16), s0[other].view(np.uint16))
    # bytes outside the group's planes and records untouched
    assert np.array_equal(page[:plane_off], before[:plane_off])
    assert np.array_equal(page[sz_off + 4 * P:], before[sz_off + 4 * P:])


def test_one_token_bytes_by_hand():
    """g=16, K side, b=2, token 1 with code 3 at coordinate 0 and code 1 at
    coordinate 8: token 1 is row 8 (hh=1); coordinate 0 -> slot 1 -> bit 4,
    coordinate 8 -> slot 3 -> bit 12; plane 0 gets bits 4 and 12, plane 1 bit 4."""
    P, g, b = 32, 16, 2
    page = np.zeros(b * P * g // 8 + 4 * P, dtype=np.uint8)
    codes = np.zeros((1, 16), np.uint8)
    codes[0, 0], codes[0, 8] = 3, 1
    oracle.pack_group_into_page(page, g, "K", P, b, 0, b * P * g // 8, np.array([1]), codes,
                                np.array([1.0], np.float16), np.array([-2.0], np.float16))
    words = page[: b * P * g // 8].view("<u4")
    plane_words = P * g // 32
    assert words[0] == (1 << 4) | (1 << 12)
    assert words[plane_words + 0] == (1 << 4)
    assert np.count_nonzero(words) == 2
    rec = page[b * P * g // 8:].view("<f2")
    assert rec[1] == 1.0 and rec[3] == -2.0 and rec[0] == 0 and rec[2] == 0


def test_section_bytes_equal_budget_accounting():
    widths = [[np.array([4, 3, 2, 2, 1, 1, 0, 0]), np.array([3, 3, 2, 1, 1, 0, 0, 0])],
              [np.array([8, 0, 0, 0, 0, 0, 0, 0]), np.array([0] * 8)]]
    P, g = 64, 16
    lay = oracle.page_layout(widths, g, P)
    bits = sum(g * int(b) + 32 for hw in widths for s in hw for b in s if b > 0)
    assert lay["page_bytes"] == P * bits // 8
    assert lay["groups"][(1, 1)] == []
    assert all(off % 16 == 0 for lst in lay["groups"].values() for (_, off, sz, _) in lst)


# --- the fragment contract the decode kernel relies on ------------------------
# PTX ISA, "Matrix fragments for mma.m16n8k16 / m16n8k8" (floating point A):
# lane -> (groupID = lane >> 2, t4 = lane % 4); element i of the A fragment sits at
# row = groupID + 8 * ((i >> 1) & 1), col = 2 t4 + (i & 1) + 8 * (i >> 2) (k16);
# for m16n8k8 only i < 4 exist.  Registers hold element pairs (2j, 2j+1).

def _frag_a(lane, i):
    gid, t4 = lane >> 2, lane & 3
    return gid + 8 * ((i >> 1) & 1), 2 * t4 + (i & 1) + 8 * (i >> 2)


def _rotr(x, n):
    n %= 32
    return ((x >> n) | (x << (32 - n))) & 0xFFFFFFFF


def _nibbles(words_by_plane, gid, t4, b):
    """Kernel recipe: R = OR_p rotr(W_p[gid], t4 - p) & (0x11111111 << p) per
    nibble plane group (planes 0-3 low accumulator, 4-7 high accumulator)."""
    lo = hi = 0
    for p in range(b):
        w = int(words_by_plane[p][gid])
        pp = p % 4
        v = _rotr(w, t4 - pp) & (0x11111111 << pp)
        if p < 4:
            lo |= v
        else:
            hi |= v
    return [((lo >> (4 * s)) & 0xF) | (((hi >> (4 * s)) & 0xF) << 4) for s in range(8)]


@pytest.mark.parametrize("g", [8, 16])
@pytest.mark.parametrize("side", ["K", "V"])
@pytest.mark.parametrize("b", [1, 3, 8])
def test_layout_feeds_mma_fragments(g, side, b):
    rng = np.random.default_rng(7 * g + b + (side == "V"))
    tb = oracle.tokens_per_block(g)
    P = 32
    page = np.zeros(b * P * g // 8 + 4 * P, dtype=np.uint8)
    codes = rng.integers(0, 2 ** b, size=(P, g)).astype(np.uint8)
    oracle.pack_group_into_page(page, g, side, P, b, 0, b * P * g // 8, np.arange(P), codes,
                                np.zeros(P, np.float16), np.zeros(P, np.float16))
    words = page[: b * P * g // 8].view("<u4").reshape(b, P // tb, 8)
    for blk in range(P // tb):
        for lane in range(32):
            gid, t4 = lane >> 2, lane & 3
            nib = _nibbles([words[p, blk] for p in range(b)], gid, t4, b)
            # register r holds the element pair (slot r, slot r + 4); see layout rules
            for mi in range(2 if g == 8 else 1):
                n_elem = 8 if (g == 16 or side == "V") else 4
                for i in range(n_elem):
                    row, col = _frag_a(lane, i)
                    if g == 16:
                        slot = ((i >> 1) & 1) + 2 * (i >> 2) + 4 * (i & 1)
                        if side == "K":
                            tok = 2 * row if row < 8 else 2 * (row - 8) + 1
                            coord = col
                        else:
                            tok, coord = col, row
                    elif side == "K":  # g = 8, m16n8k8 per 16-token half mi
                        slot = ((i >> 1) & 1) + 2 * mi + 4 * (i & 1)
                        r = row
                        tok = 16 * mi + (2 * r if r < 8 else 2 * (r - 8) + 1)
                        coord = col
                    else:  # g = 8, V: m16n8k16 with rows 8..15 zero padding
                        if row >= 8:
                            continue
                        slot = mi + 2 * (i >> 2) + 4 * (i & 1)
                        tok, coord = 16 * mi + col, row
                    assert nib[slot] == codes[blk * tb + tok, coord]
