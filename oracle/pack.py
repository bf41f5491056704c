"""Bit packing of integer codes into 32-bit words, as the packed-cache layout states.

row layout   : per token row, channel c in word c // (32/b) at bit b * (c % (32/b)),
               least significant bits first.
pair layout  : tokens 2u and 2u+1 share words; word w holds (16/b) channels of token
               2u in bits 0..15 and the same channels of token 2u+1 in bits 16..31.
3-bit planes : the low two bits of every code in the row layout, then the high bit
               in a 1-bit row layout.

Pinned by tests/test_oracle_pack.py (pack / unpack round trip of every code value at
every lane position, and hand-written words).
"""
from __future__ import annotations

import numpy as np


def pack_row(codes, bits):
    """codes [..., n] (n a multiple of 32/bits) -> uint32 [..., n * bits / 32]."""
    codes = np.asarray(codes, np.uint64)
    per = 32 // bits
    n = codes.shape[-1]
    assert n % per == 0
    c = codes.reshape(codes.shape[:-1] + (n // per, per))
    shifts = (np.arange(per, dtype=np.uint64) * np.uint64(bits))
    words = (c << shifts).sum(axis=-1)
    return words.astype(np.uint32)


def unpack_row(words, bits, n):
    words = np.asarray(words, np.uint64)
    per = 32 // bits
    shifts = (np.arange(per, dtype=np.uint64) * np.uint64(bits))
    c = (words[..., None] >> shifts) & np.uint64((1 << bits) - 1)
    return c.reshape(words.shape[:-1] + (words.shape[-1] * per,))[..., :n].astype(np.int64)


def pack_pair(codes, bits):
    """codes [n_tokens, D] -> uint32 [ceil(n_tokens/2), D * bits / 16]."""
    codes = np.asarray(codes, np.uint64)
    n, D = codes.shape
    per = 16 // bits
    assert D % per == 0
    if n % 2:
        codes = np.concatenate([codes, np.zeros((1, D), np.uint64)], axis=0)
    shifts = (np.arange(per, dtype=np.uint64) * np.uint64(bits))
    halves = (codes.reshape(-1, 2, D // per, per) << shifts).sum(axis=-1)  # [pairs, 2, W]
    words = halves[:, 0, :] | (halves[:, 1, :] << np.uint64(16))
    return words.astype(np.uint32)


def unpack_pair(words, bits, n_tokens, D):
    words = np.asarray(words, np.uint64)
    per = 16 // bits
    shifts = (np.arange(per, dtype=np.uint64) * np.uint64(bits))
    mask = np.uint64((1 << bits) - 1)
    lo = (words[..., None] >> shifts) & mask
    hi = (words[..., None] >> (shifts + np.uint64(16))) & mask
    pairs = words.shape[0]
    out = np.stack([lo.reshape(pairs, D), hi.reshape(pairs, D)], axis=1).reshape(2 * pairs, D)
    return out[:n_tokens].astype(np.int64)


def pack_3bit(codes):
    """codes [..., D] in 0..7 -> uint32 [..., 3D/32]: low-2-bit plane then high-bit plane."""
    codes = np.asarray(codes, np.int64)
    lo = pack_row(codes & 3, 2)
    hi = pack_row(codes >> 2, 1)
    return np.concatenate([lo, hi], axis=-1)


def unpack_3bit(words, D):
    words = np.asarray(words)
    lo = unpack_row(words[..., : D // 16], 2, D)
    hi = unpack_row(words[..., D // 16:], 1, D)
    return lo | (hi << 2)
