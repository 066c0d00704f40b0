"""Pins of the oracle's page layout: bijection, hand-derived addresses, round trip,
byte accounting, and that the layout feeds the sm_80+ ``mma.sync`` A-operand
fragments through the nibble extraction the decode kernel performs."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_rows():
    with open(os.path.join(GOLDEN, "layout_bits.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                yield [x.strip() for x in line.split("|")]


@pytest.mark.parametrize("b", [1, 2, 3, 4, 8])
def test_addresses_are_a_bijection(b):
    for g in (8, 16):
        for side in ("K", "V"):
            tb = oracle.tokens_per_block(g)
            seen = {oracle.code_bit_address(g, side, b, t, k, p)
                    for t in range(tb) for k in range(g) for p in range(b)}
            assert len(seen) == 256 * b
            assert all(0 <= w < 8 * b and 0 <= bit < 32 for w, bit in seen)


def test_fragment_positions_are_a_bijection():
    for g in (8, 16):
        for side in ("K", "V"):
            tb = oracle.tokens_per_block(g)
            seen = {oracle.fragment_position(g, side, t, k) for t in range(tb) for k in range(g)}
            assert len(seen) == 256
            assert all(0 <= gid < 8 and 0 <= t4 < 4 and 0 <= sl < 8 for gid, t4, sl in seen)


def test_hand_derived_addresses():
    rows = [r for r in _golden_rows() if r[0] != "rec"]
    assert len(rows) >= 10
    for r in rows:
        g, side, b, tau, k, p, word, bit = int(r[0]), r[1], *map(int, r[2:])
        assert oracle.code_bit_address(g, side, b, tau, k, p) == (word, bit), r


def test_hand_derived_record_indices():
    rows = [r for r in _golden_rows() if r[0] == "rec"]
    assert rows
    for r in rows:
        P, tau, idx = map(int, r[1:])
        assert oracle.record_index(P, tau) == idx, r
    # the records of a page are a permutation of its token pairs
    for P in (32, 64, 96):
        assert sorted(oracle.record_index(P, 2 * u) for u in range(P // 2)) == list(range(P // 2))


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
    """g=16, K side, b=2, P=32, token 1 with code 3 at coordinate 0 and code 1 at
    coordinate 8.  Token 1 is row 8 (gid 0, hh 1); coordinate 0 has t4 0, ch 0 ->
    slot 1; coordinate 8 has t4 0, ch 1 -> slot 3.  b=2 puts lane (0, 0) in word 0
    at nibble bits 0-1: code 3 -> bits 4, 5; code 1 -> bit 12.  Token 1 is in pair
    0, record 0: s at fp16 index 1, z at index 3."""
    P, g, b = 32, 16, 2
    page = np.zeros(b * P * g // 8 + 4 * P, dtype=np.uint8)
    codes = np.zeros((1, 16), np.uint8)
    codes[0, 0], codes[0, 8] = 3, 1
    oracle.pack_group_into_page(page, g, "K", P, b, 0, b * P * g // 8, np.array([1]), codes,
                                np.array([1.0], np.float16), np.array([-2.0], np.float16))
    words = page[: b * P * g // 8].view("<u4")
    assert words[0] == (1 << 4) | (1 << 5) | (1 << 12)
    assert np.count_nonzero(words) == 1
    rec = page[b * P * g // 8:].view("<f2")
    assert rec[1] == 1.0 and rec[3] == -2.0 and rec[0] == 0 and rec[2] == 0
    assert np.count_nonzero(rec) == 2


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


def _slot_codes(block_words, gid, t4, b):
    """Kernel recipe: this lane's 8 codes (slot order) from one block, by width.
    b <= 4: one 32-bit word of nibbles, x; slot s is (x >> 4 s) & (2^b - 1)."""
    w = [int(v) for v in block_words]
    lane = 4 * gid + t4
    if b == 8:
        w0, w1 = w[2 * lane], w[2 * lane + 1]
        byte = lambda x, i: (x >> (8 * i)) & 0xFF
        return [byte(w0, 0), byte(w0, 1), byte(w1, 0), byte(w1, 1),
                byte(w0, 2), byte(w0, 3), byte(w1, 2), byte(w1, 3)]
    if b == 4:
        x = w[lane]
    elif b == 2:
        x = w[2 * gid + t4 // 2] >> (2 * (t4 % 2))
    elif b == 1:
        x = w[gid] >> t4
    else:  # b == 3
        lo = w[2 * gid + t4 // 2] >> (2 * (t4 % 2))
        hi = _rotr(w[16 + gid], t4 - 2)
        x = (lo & 0x33333333) | (hi & 0xCCCCCCCC)
    return [(x >> (4 * s)) & ((1 << b) - 1) for s in range(8)]


@pytest.mark.parametrize("g", [8, 16])
@pytest.mark.parametrize("side", ["K", "V"])
@pytest.mark.parametrize("b", [1, 2, 3, 4, 8])
def test_layout_feeds_mma_fragments(g, side, b):
    rng = np.random.default_rng(7 * g + b + (side == "V"))
    tb = oracle.tokens_per_block(g)
    P = 64
    page = np.zeros(b * P * g // 8 + 4 * P, dtype=np.uint8)
    codes = rng.integers(0, 2 ** b, size=(P, g)).astype(np.uint8)
    oracle.pack_group_into_page(page, g, side, P, b, 0, b * P * g // 8, np.arange(P), codes,
                                np.zeros(P, np.float16), np.zeros(P, np.float16))
    words = page[: b * P * g // 8].view("<u4").reshape(P // tb, 8 * b)
    for blk in range(P // tb):
        for lane in range(32):
            gid, t4 = lane >> 2, lane & 3
            nib = _slot_codes(words[blk], gid, t4, b)
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


def test_records_feed_the_kernels_lanes():
    """With P/16 tiles per page, the lane reading token pair j of tiles
    t0 .. t0+3 finds them in 4 consecutive records starting at j*(P/16) + t0."""
    P = 64
    blocks = P * 16 // 8  # b = 1
    page = np.zeros(blocks + 4 * P, dtype=np.uint8)
    s = (np.arange(P) + 1).astype(np.float16)
    oracle.pack_group_into_page(page, 16, "K", P, 1, 0, blocks, np.arange(P), np.zeros((P, 16), np.uint8), s,
                                -s)
    rec = page[blocks:].view("<f2").reshape(P // 2, 4)
    for j in range(8):
        for t in range(P // 16):
            r = rec[j * (P // 16) + t]
            tok = 16 * t + 2 * j
            assert (r[0], r[1], r[2], r[3]) == (s[tok], s[tok + 1], -s[tok], -s[tok + 1])
