"""Bit packing of integer codes into int32 words (oracle side).

TEST INFRASTRUCTURE ONLY (see the package docstring).

"[SGLang] AutoRound: 자동 라운딩 최적화 양자화", section "1. AutoRoundConfig":
codes of ``bits`` bits are packed into 32-bit words with
pack_factor = Fraction(32, bits), exact also for 3 bits, where codes straddle
word boundaries.  The page gives the ratio only; reading used here: each row is
one little-endian bit stream along the last dimension -- bit j of code i (row-
local index) is global bit i*bits + j of the row, i.e. bit (i*bits + j) mod 32
of word (i*bits + j) // 32.  Rows pack independently.

Written as a plain per-code loop over Python integers so it can be checked by
eye; only meant for test-sized inputs.
"""
from __future__ import annotations

import numpy as np


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    codes = np.asarray(codes)
    rows, cols = codes.shape
    if (cols * bits) % 32:
        raise ValueError("cols * bits must be a multiple of 32")
    words = cols * bits // 32
    out = np.zeros((rows, words), dtype=np.uint32)
    for r in range(rows):
        stream = 0
        for i in range(cols):
            c = int(codes[r, i])
            if c < 0 or c >= (1 << bits):
                raise ValueError("code out of range")
            stream |= c << (i * bits)
        for w in range(words):
            out[r, w] = (stream >> (32 * w)) & 0xFFFFFFFF
    return out.view(np.int32)


def unpack_codes(packed: np.ndarray, bits: int, cols: int) -> np.ndarray:
    packed = np.asarray(packed).view(np.uint32)
    rows, words = packed.shape
    out = np.zeros((rows, cols), dtype=np.uint8)
    for r in range(rows):
        stream = 0
        for w in range(words):
            stream |= int(packed[r, w]) << (32 * w)
        for i in range(cols):
            out[r, i] = (stream >> (i * bits)) & ((1 << bits) - 1)
    return out
