"""Greedy residual encoder of one new key / value into codes (CPU oracle).

TEST INFRASTRUCTURE ONLY (see cvq_oracle.py).  The pages encode with a learned encoder
(CommVQ abstract; summary page "Approach"), which needs trained weights; this is the plain
stand-in: additive quantization by greedy residual rounds (review page, "key_machinery":
R residual rounds refine the reconstruction).  For each group and round r = 0..R-1 pick
the codeword nearest to the current residual, then subtract it.

Because a floating-point comparison decides an integer code, the decision is taken in
float32 with a fixed order, the same as the kernel's:
    dist(c) = (((x_0 - c_0)^2 + (x_1 - c_1)^2) + ...) + (x_7 - c_7)^2,
every subtraction, square and addition rounded to float32 (no fused multiply-add), and ties
go to the smallest code index.  Keys are encoded before RoPE (the cache stores pre-RoPE
keys, as the decode path expects); a key group is its 4 pairs as 8 floats (re, im, ...).
"""
from __future__ import annotations

import numpy as np

N_GROUPS = 16


def _dist32(x: np.ndarray, cands: np.ndarray) -> np.ndarray:
    """float32 squared distances of x [8] to each row of cands [N, 8], summed in order."""
    x = x.astype(np.float32)
    cands = cands.astype(np.float32)
    acc = np.zeros(cands.shape[0], dtype=np.float32)
    for d in range(8):
        diff = np.float32(x[d]) - cands[:, d]          # float32
        acc = (acc + (diff * diff).astype(np.float32)).astype(np.float32)
    return acc


def encode_group(x: np.ndarray, cb_rounds: np.ndarray):
    """Codes [R] and the float32 residual for one group vector x [8] against codebooks
    cb_rounds [R, 256, 8] (float32)."""
    res = np.asarray(x, dtype=np.float32).copy()
    codes = []
    for r in range(cb_rounds.shape[0]):
        d = _dist32(res, cb_rounds[r])
        c = int(np.argmin(d))                           # first index on ties
        codes.append(c)
        res = (res - cb_rounds[r, c].astype(np.float32)).astype(np.float32)
    return codes, res


def encode_vector(v: np.ndarray, cb_h: np.ndarray) -> np.ndarray:
    """Codes [R, 16] (uint8) of one 128-dim vector against one head's codebook, viewed as
    [16, R, 256, 8] (a key codebook [16, R, 256, 4, 2] is reshaped to that)."""
    cb = np.asarray(cb_h, dtype=np.float32)
    R = cb.shape[1]
    cb = cb.reshape(N_GROUPS, R, 256, 8)
    out = np.zeros((R, N_GROUPS), dtype=np.uint8)
    v = np.asarray(v, dtype=np.float32).reshape(N_GROUPS, 8)
    for g in range(N_GROUPS):
        codes, _ = encode_group(v[g], cb[g])
        out[:, g] = codes
    return out


def encode_append(keys, values, key_cb, val_cb, positions, key_codes, val_codes):
    """Write the codes of keys / values [B, Hkv, 128] at position positions[b] of the code
    buffers [B, Hkv, T_cap, R, 16] (in place); positions outside [0, T_cap) are skipped."""
    B, Hkv, _ = keys.shape
    T = key_codes.shape[2]
    for b in range(B):
        p = int(positions[b])
        if p < 0 or p >= T:
            continue
        for h in range(Hkv):
            key_codes[b, h, p] = encode_vector(keys[b, h], key_cb[h])
            val_codes[b, h, p] = encode_vector(values[b, h], val_cb[h])
    return key_codes, val_codes
