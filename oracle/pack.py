"""6-bit code packing of the paper's parameterization (CPU oracle).

TEST INFRASTRUCTURE ONLY (see cvq_oracle.py).  With 64 codewords per (group, round) a code
has 6 bits (CommVQ summary page, "Key results": R = 11 rounds of 64-entry codebooks over
64-scalar groups is the 1.03-bit setting, 11 x 6 / 64 bits per scalar).  Stored one per
byte, the code stream carries 8 / 6 of that; packed, it carries exactly that.  The pages do
not fix a bit layout; this one is plain little-endian:

    along a row of codes (one (sequence, KV head, group, round) row of the planar layout),
    codes t = 4i .. 4i+3 form the 24-bit little-endian word held in bytes 3i .. 3i+2, code
    4i + j occupying bits 6j .. 6j+5 of that word.

So a row of n codes (n a multiple of 4) takes 3n/4 bytes.  Only the low 6 bits of an input
byte are packed (the unpacked layout ignores the top 2 bits of every code byte).
"""
from __future__ import annotations

import numpy as np


def pack_codes6(codes: np.ndarray) -> np.ndarray:
    """Pack uint8 codes [..., n] (n % 4 == 0) into uint8 [..., 3n/4]."""
    c = np.asarray(codes, dtype=np.uint8)
    n = c.shape[-1]
    if n % 4:
        raise ValueError("row length must be a multiple of 4")
    lead = c.shape[:-1]
    flat = c.reshape(-1, n)
    out = np.zeros((flat.shape[0], 3 * n // 4), dtype=np.uint8)
    for i in range(n // 4):
        word = np.zeros(flat.shape[0], dtype=np.uint32)
        for j in range(4):
            word |= (flat[:, 4 * i + j].astype(np.uint32) & 63) << (6 * j)
        out[:, 3 * i + 0] = word & 0xFF
        out[:, 3 * i + 1] = (word >> 8) & 0xFF
        out[:, 3 * i + 2] = (word >> 16) & 0xFF
    return out.reshape(*lead, 3 * n // 4)


def unpack_codes6(packed: np.ndarray, n: int) -> np.ndarray:
    """Inverse of pack_codes6: uint8 [..., 3n/4] -> codes uint8 [..., n] (values 0..63)."""
    p = np.asarray(packed, dtype=np.uint8)
    if n % 4 or p.shape[-1] != 3 * n // 4:
        raise ValueError("packed row must hold 3n/4 bytes, n a multiple of 4")
    lead = p.shape[:-1]
    flat = p.reshape(-1, p.shape[-1])
    out = np.zeros((flat.shape[0], n), dtype=np.uint8)
    for i in range(n // 4):
        word = (flat[:, 3 * i].astype(np.uint32) | (flat[:, 3 * i + 1].astype(np.uint32) << 8)
                | (flat[:, 3 * i + 2].astype(np.uint32) << 16))
        for j in range(4):
            out[:, 4 * i + j] = (word >> (6 * j)) & 63
    return out.reshape(*lead, n)
