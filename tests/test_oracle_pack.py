"""Pins of oracle.pack: hand-written words and an exhaustive round trip of every code
value at every lane position."""
import numpy as np
import pytest

from oracle import pack


def test_row_layout_by_hand():
    # 4-bit: channel c at bits 4*(c % 8) of word c // 8
    codes = np.arange(16) % 16
    w = pack.pack_row(codes, 4)
    assert w.tolist() == [0x76543210, 0xFEDCBA98]
    # 2-bit: channel c at bits 2*(c % 16)
    codes = np.array([1, 2, 3, 0] * 4)
    assert pack.pack_row(codes, 2).tolist() == [0x39393939]
    # 1-bit
    codes = np.zeros(32, int)
    codes[0] = codes[31] = 1
    assert pack.pack_row(codes, 1).tolist() == [0x80000001]


def test_pair_layout_by_hand():
    # 2-bit values, D = 8: one word per pair; token 2u in the low half
    a = np.array([3] + [0] * 7)
    b = np.array([0] * 7 + [2])
    w = pack.pack_pair(np.stack([a, b]), 2)
    assert w.tolist() == [[0x80000003]]
    # odd count: the missing token's half is zero
    w = pack.pack_pair(np.stack([a, b, a]), 2)
    assert w.tolist() == [[0x80000003], [0x00000003]]


@pytest.mark.parametrize("bits", [1, 2, 4])
def test_row_roundtrip_exhaustive(bits):
    per = 32 // bits
    for pos in range(per):
        for v in range(2 ** bits):
            codes = np.zeros(per * 2, int)
            codes[pos] = v
            codes[per + (per - 1 - pos)] = v
            w = pack.pack_row(codes, bits)
            assert (int(w[0]) >> (bits * pos)) & ((1 << bits) - 1) == v
            np.testing.assert_array_equal(pack.unpack_row(w, bits, per * 2), codes)


@pytest.mark.parametrize("bits", [2, 4])
def test_pair_roundtrip_exhaustive(bits):
    D = 32
    per = 16 // bits
    for pos in range(D):
        for v in range(2 ** bits):
            codes = np.zeros((2, D), int)
            codes[0, pos] = v
            codes[1, D - 1 - pos] = (v + 1) % (2 ** bits)
            w = pack.pack_pair(codes, bits)
            word = int(w[0, pos // per])
            assert (word >> (bits * (pos % per))) & ((1 << bits) - 1) == v
            np.testing.assert_array_equal(pack.unpack_pair(w, bits, 2, D), codes)


def test_3bit_planes_roundtrip():
    r = np.random.default_rng(0)
    codes = r.integers(0, 8, (5, 128))
    w = pack.pack_3bit(codes)
    assert w.shape == (5, 12)
    np.testing.assert_array_equal(pack.unpack_3bit(w, 128), codes)
    # the high-bit plane holds bit 2 of channel c at bit c % 32 of word 8 + c // 32
    c = 77
    assert ((int(w[0, 8 + c // 32]) >> (c % 32)) & 1) == (codes[0, c] >> 2)
