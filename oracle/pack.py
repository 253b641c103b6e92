"""Bit packing of integer codes (oracle; test infrastructure only).

The pages only say that weights become b-bit integers (GPTQ encyclopedia
article: 4-bit weights cut memory to a quarter; 2- and 3-bit are supported).
Storage convention taken here: along each row, code j occupies bits
[j*b, j*b + b) of one continuous little-endian bit stream, cut into 32-bit
words, least significant bit first. A row of n codes takes n*b/32 words
(n*b must be a multiple of 32). Codes may straddle two words when 32 % b != 0.
"""
from __future__ import annotations

import numpy as np


def pack_codes(codes, bits: int) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint64)
    m, n = codes.shape
    assert (n * bits) % 32 == 0
    words = np.zeros((m, n * bits // 32), dtype=np.uint64)
    for j in range(n):
        for b in range(bits):
            p = j * bits + b
            words[:, p // 32] |= ((codes[:, j] >> np.uint64(b)) & np.uint64(1)) << np.uint64(p % 32)
    return words.astype(np.uint32)


def unpack_codes(words, bits: int, n: int) -> np.ndarray:
    words = np.asarray(words, dtype=np.uint64)
    m = words.shape[0]
    codes = np.zeros((m, n), dtype=np.uint64)
    for j in range(n):
        for b in range(bits):
            p = j * bits + b
            codes[:, j] |= ((words[:, p // 32] >> np.uint64(p % 32)) & np.uint64(1)) << np.uint64(b)
    return codes.astype(np.int64)
