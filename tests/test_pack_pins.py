"""Pins of the oracle's 6-bit code packer (oracle/pack.py), independent of the packer:
bytes worked out by hand from the stated layout (code 4i + j at bits 6j .. 6j+5 of the
little-endian 24-bit word in bytes 3i .. 3i+2), single-code positions, round trips, sizes,
and a planted mistake (big-endian words) that the hand-worked bytes catch."""
import numpy as np
import pytest

from oracle import pack as P


def test_hand_worked_bytes():
    # [1, 2, 3, 63]: 1 + (2 << 6) + (3 << 12) + (63 << 18) = 1 + 128 + 12288 + 16515072
    # = 16527489 = 0xFC3081 -> bytes 0x81, 0x30, 0xFC
    assert P.pack_codes6(np.array([1, 2, 3, 63], np.uint8)).tolist() == [0x81, 0x30, 0xFC]
    # [5, 40, 17, 9]: 5 + 40*64 + 17*4096 + 9*262144 = 5 + 2560 + 69632 + 2359296 = 2431493
    # = 0x251A05 -> 0x05, 0x1A, 0x25
    assert P.pack_codes6(np.array([5, 40, 17, 9], np.uint8)).tolist() == [0x05, 0x1A, 0x25]


@pytest.mark.parametrize("j, expect", [(0, [0x3F, 0, 0]), (1, [0xC0, 0x0F, 0]),
                                       (2, [0, 0xF0, 0x03]), (3, [0, 0, 0xFC])])
def test_single_code_bit_positions(j, expect):
    # code 63 (all six bits) in slot j sits at bits 6j .. 6j+5 of the 24-bit word
    c = np.zeros(4, np.uint8)
    c[j] = 63
    assert P.pack_codes6(c).tolist() == expect


def test_top_two_bits_ignored_and_sizes():
    c = np.array([0xC1, 0x80, 0x7F, 0x40], np.uint8)      # low 6 bits: 1, 0, 63, 0
    assert P.pack_codes6(c).tolist() == P.pack_codes6(np.array([1, 0, 63, 0], np.uint8)).tolist()
    assert P.pack_codes6(np.zeros((2, 3, 64), np.uint8)).shape == (2, 3, 48)
    with pytest.raises(ValueError):
        P.pack_codes6(np.zeros(6, np.uint8))


def test_round_trip_random_rows():
    rng = np.random.default_rng(7)
    c = rng.integers(0, 64, size=(3, 2, 5, 128), dtype=np.uint8)
    p = P.pack_codes6(c)
    assert p.shape == (3, 2, 5, 96)
    assert np.array_equal(P.unpack_codes6(p, 128), c)
    # bits of one code never leak into a neighbour: changing one code changes <= 2 bytes
    c2 = c.copy()
    c2[1, 1, 2, 37] ^= 63
    diff = np.nonzero(P.pack_codes6(c2) != p)
    assert len(set(zip(*diff))) <= 2 and set(diff[3]) <= {27, 28}


def test_planted_big_endian_mistake_is_caught(monkeypatch):
    def big_endian(codes):
        c = np.asarray(codes, np.uint8)
        out = []
        for i in range(c.shape[-1] // 4):
            w = 0
            for j in range(4):
                w |= (int(c[4 * i + j]) & 63) << (6 * j)
            out += [(w >> 16) & 255, (w >> 8) & 255, w & 255]
        return np.array(out, np.uint8)
    monkeypatch.setattr(P, "pack_codes6", big_endian)
    with pytest.raises(AssertionError):
        test_hand_worked_bytes()
