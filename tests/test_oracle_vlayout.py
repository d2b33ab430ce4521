"""Pins of the oracle's 3-bit V tile layout (the packed format of V codes in a page).

The layout is this build's own (the method's pages fix no bit packing): a page's V region
holds 16-token blocks in which each 12-byte group carries the codes of four tokens' eight
dims, so that a 16-bit half of a word is four tokens' codes of one dim.  These tests pin
the oracle's implementation of it against (1) examples worked out by hand from the
layout's written definition (tests/golden/v_tile_layout_examples.txt), (2) a bijection
between (slot, dim, code bit) and the bits of the region, and (3) the round trip.  The K
codes and the 2- and 4-bit V codes keep one record per token (pinned elsewhere).
"""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "v_tile_layout_examples.txt")


def _examples():
    out = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        lhs, rhs = line.split("|")
        d, slot, dim, code = (int(x) for x in lhs.split())
        expect = {}
        for item in rhs.split():
            b, v = item.split(":")
            expect[int(b)] = int(v, 16)
        out.append((d, slot, dim, code, expect))
    return out


@pytest.mark.parametrize("case", _examples(), ids=lambda c: f"d{c[0]}_s{c[1]}_i{c[2]}_c{c[3]}")
def test_hand_worked_bit_positions(oracle, case):
    d, slot, dim, code, expect = case
    region = np.zeros(64 * 3 * d // 8, np.uint8)
    codes = np.zeros(d, np.uint8)
    codes[dim] = code
    oracle.v_put_codes(region, slot, codes)
    nz = {int(i): int(region[i]) for i in np.nonzero(region)[0]}
    assert nz == expect
    assert oracle.v_get_codes(region, slot, d)[dim] == code


@pytest.mark.parametrize("d", [128, 256])
def test_every_code_bit_has_its_own_region_bit(oracle, d):
    """Writing code 7 (all three bits) at one (slot, dim) sets exactly three bits; over all
    (slot, dim) those bit sets are disjoint and cover the region: the layout is a
    bijection, 48 (96) bytes per token as the format requires."""
    nbytes = 64 * 3 * d // 8
    seen = np.zeros(nbytes * 8, bool)
    for slot in range(64):
        for dim in range(d):
            region = np.zeros(nbytes, np.uint8)
            codes = np.zeros(d, np.uint8)
            codes[dim] = 7
            oracle.v_put_codes(region, slot, codes)
            bits = np.nonzero(np.unpackbits(region, bitorder="little"))[0]
            assert len(bits) == 3
            assert not seen[bits].any()
            seen[bits] = True
    assert seen.all()


@pytest.mark.parametrize("d", [128, 256])
def test_round_trip_and_overwrite(oracle, d):
    rng = np.random.default_rng(d)
    nbytes = 64 * 3 * d // 8
    region = np.zeros(nbytes, np.uint8)
    codes = rng.integers(0, 8, (64, d)).astype(np.uint8)
    for s in rng.permutation(64):
        oracle.v_put_codes(region, int(s), codes[s])
    back = np.stack([oracle.v_get_codes(region, s, d) for s in range(64)])
    assert np.array_equal(back, codes)
    # rewriting one slot changes that slot only
    new = rng.integers(0, 8, d).astype(np.uint8)
    oracle.v_put_codes(region, 37, new)
    codes[37] = new
    back = np.stack([oracle.v_get_codes(region, s, d) for s in range(64)])
    assert np.array_equal(back, codes)
    # the record view agrees with the record packing of the same codes
    rec = oracle.v_region_records(region, d)
    for s in (0, 15, 16, 37, 63):
        assert np.array_equal(rec[s], oracle.pack_codes(codes[s]))


def test_half_words_are_one_dim_of_four_tokens(oracle):
    """The property the decoder relies on: the low 16 bits of word b of group (block B,
    quad t, unit u) are, nibble j, the code of slot 16B + 2t + (j & 1) + 8(j >> 1) at dim
    8u + 2b; the high 16 bits the same slots at dim 8u + 2b + 1 (3-bit nibbles)."""
    d = 128
    rng = np.random.default_rng(5)
    region = np.zeros(64 * 48, np.uint8)
    codes = rng.integers(0, 8, (64, d)).astype(np.uint8)
    for s in range(64):
        oracle.v_put_codes(region, s, codes[s])
    words = region.view("<u4")
    for B in range(4):
        for t in range(4):
            for u in range(16):
                g = (B * 6 * d + ((u >> 1) * 8 + 2 * t + (u & 1)) * 12) // 4
                slots = [16 * B + 2 * t + (j & 1) + 8 * (j >> 1) for j in range(4)]
                for b in range(3):
                    w = int(words[g + b])
                    for j in range(4):
                        assert (w >> (4 * j)) & 7 == codes[slots[j], 8 * u + 2 * b]
                        assert (w >> (16 + 4 * j)) & 7 == codes[slots[j], 8 * u + 2 * b + 1]
