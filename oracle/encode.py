"""Greedy residual encoder of one new key / value into codes (CPU oracle).

TEST INFRASTRUCTURE ONLY (see cvq_oracle.py).  The pages encode with a learned encoder
(CommVQ abstract; summary page "Approach"), which needs trained weights; this is the plain
stand-in: additive quantization by greedy residual rounds (review page, "key_machinery":
R residual rounds refine the reconstruction).  For each group and round r = 0..R-1 pick
the codeword nearest to the current residual, then subtract it.

Because a floating-point comparison decides an integer code, the decision is taken in
float32 with a fixed order, the same as the kernel's:
    dist(c) = (((x_0 - c_0)^2 + (x_1 - c_1)^2) + ...) + (x_{D-1} - c_{D-1})^2,
every subtraction, square and addition rounded to float32 (no fused multiply-add), and ties
go to the smallest code index.  Keys are encoded before RoPE (the cache stores pre-RoPE
keys, as the decode path expects); a key group is its pairs as floats (re, im, ...).
Both layouts of the decode path are covered, read off the codebook shape: 16 groups of
D = 8 scalars with 256 codewords, or 2 groups of D = 64 scalars with 64 codewords (the
paper's own parameterization); codes are [R, NG] per vector.
"""
from __future__ import annotations

import numpy as np

def _dist32(x: np.ndarray, cands: np.ndarray) -> np.ndarray:
    """float32 squared distances of x [D] to each row of cands [N, D], summed in order."""
    x = x.astype(np.float32)
    cands = cands.astype(np.float32)
    acc = np.zeros(cands.shape[0], dtype=np.float32)
    for d in range(cands.shape[1]):
        diff = np.float32(x[d]) - cands[:, d]          # float32
        acc = (acc + (diff * diff).astype(np.float32)).astype(np.float32)
    return acc


def encode_group(x: np.ndarray, cb_rounds: np.ndarray):
    """Codes [R] and the float32 residual for one group vector x [D] against codebooks
    cb_rounds [R, N, D] (float32)."""
    res = np.asarray(x, dtype=np.float32).copy()
    codes = []
    for r in range(cb_rounds.shape[0]):
        d = _dist32(res, cb_rounds[r])
        c = int(np.argmin(d))                           # first index on ties
        codes.append(c)
        res = (res - cb_rounds[r, c].astype(np.float32)).astype(np.float32)
    return codes, res


def encode_vector(v: np.ndarray, cb_h: np.ndarray) -> np.ndarray:
    """Codes [R, NG] (uint8) of one 128-dim vector against one head's codebook, viewed as
    [NG, R, N, D] with NG * D = 128 (a key codebook [NG, R, N, PPG, 2] is reshaped to that)."""
    cb = np.asarray(cb_h, dtype=np.float32)
    n_groups, R, n_codes = cb.shape[0], cb.shape[1], cb.shape[2]
    D = 128 // n_groups
    cb = cb.reshape(n_groups, R, n_codes, D)
    out = np.zeros((R, n_groups), dtype=np.uint8)
    v = np.asarray(v, dtype=np.float32).reshape(n_groups, D)
    for g in range(n_groups):
        codes, _ = encode_group(v[g], cb[g])
        out[:, g] = codes
    return out


def encode_append(keys, values, key_cb, val_cb, positions, key_codes, val_codes,
                  codes_layout="token"):
    """Write the codes of keys / values [B, Hkv, 128] at position positions[b] of the code
    buffers (in place): token-major [B, Hkv, T_cap, R, NG], or with codes_layout "planar"
    [B, Hkv, NG, R, T_cap].  Positions outside [0, T_cap) are skipped."""
    B, Hkv, _ = keys.shape
    T = key_codes.shape[4] if codes_layout == "planar" else key_codes.shape[2]
    for b in range(B):
        p = int(positions[b])
        if p < 0 or p >= T:
            continue
        for h in range(Hkv):
            kc = encode_vector(keys[b, h], key_cb[h])          # [R, NG]
            vc = encode_vector(values[b, h], val_cb[h])
            if codes_layout == "planar":
                key_codes[b, h, :, :, p] = kc.T
                val_codes[b, h, :, :, p] = vc.T
            else:
                key_codes[b, h, p] = kc
                val_codes[b, h, p] = vc
    return key_codes, val_codes
