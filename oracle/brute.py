"""Scalar pure-Python brute force of the same decode step, for tiny inputs (T <= 8).

TEST INFRASTRUCTURE ONLY (see cvq_oracle.py).  Written independently of the NumPy
oracle: explicit loops over every dimension, the `math` module, no arrays.  It pins
the NumPy oracle: the two must agree to ~1e-12.

The definition followed is the same (CommVQ review page, pith.science arXiv
2506.18879, "key_machinery"; CommVQ abstract on the aitopics.org page):
  key dim (2j + e), e in {0, 1}, pair j, group G = j // PPG, slot p = j % PPG
  (PPG pairs per group: 4 with 256-entry codebooks, 32 in the paper's 64-entry layout):
      k = sum_r key_cb[h][G][r][code][p][e]
  RoPE at position t, angle a = base^(-2j/128) * t:
      k'[2j]   = cos(a) k[2j] - sin(a) k[2j+1]
      k'[2j+1] = sin(a) k[2j] + cos(a) k[2j+1]
  s_t = sum_d q[d] k'[d] / sqrt(128)
  out[d] = sum_t softmax(s)_t * v_t[d],   v_t[VD G + d] = sum_r val_cb[h][G][r][code][d]
"""
from __future__ import annotations

import math


def brute_attend_head(q, key_cb_h, val_cb_h, key_codes, val_codes, seq_len, base):
    """q: 128 floats.  key_cb_h[G][r][c][p][e], val_cb_h[G][r][c][d] nested sequences
    (NumPy arrays index the same way).  key_codes[t][r][G], val_codes[t][r][G] ints.
    Returns (out list of 128, lse)."""
    if seq_len == 0:
        return [0.0] * 128, -math.inf
    R = len(key_codes[0])
    ppg = len(key_cb_h[0][0][0])      # pairs per key group
    vd = len(val_cb_h[0][0][0])       # dims per value group
    s = []
    vals = []
    for t in range(seq_len):
        key = [0.0] * 128
        for d in range(128):
            j, e = divmod(d, 2)
            G, p = divmod(j, ppg)
            acc = 0.0
            for r in range(R):
                acc += float(key_cb_h[G][r][int(key_codes[t][r][G])][p][e])
            key[d] = acc
        dot = 0.0
        for j in range(64):
            a = (float(base) ** (-2.0 * j / 128.0)) * t
            x, y = key[2 * j], key[2 * j + 1]
            rx = math.cos(a) * x - math.sin(a) * y
            ry = math.sin(a) * x + math.cos(a) * y
            dot += float(q[2 * j]) * rx + float(q[2 * j + 1]) * ry
        s.append(dot / math.sqrt(128.0))
        v = [0.0] * 128
        for d in range(128):
            G, dd = divmod(d, vd)
            acc = 0.0
            for r in range(R):
                acc += float(val_cb_h[G][r][int(val_codes[t][r][G])][dd])
            v[d] = acc
        vals.append(v)
    m = max(s)
    e = [math.exp(x - m) for x in s]
    tot = math.fsum(e)
    out = [0.0] * 128
    for t in range(seq_len):
        wt = e[t] / tot
        for d in range(128):
            out[d] += wt * vals[t][d]
    return out, m + math.log(tot)
