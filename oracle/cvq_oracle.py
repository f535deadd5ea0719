"""Float64 CPU oracle for CommVQ decode attention over a vector-quantized KV cache.

TEST INFRASTRUCTURE ONLY. Nothing in the library's product path imports, links or
runs this module; only the tests, the smoke check and the benchmark's CPU-baseline
leg use it.  It shares no code with the CUDA path.

What it computes is the plain definition of one decode step of attention, written
out step by step (NumPy float64, no blocking, fusion or reordering beyond what the
definition states):

  1. theta_j = base^(-2j/128), j = 0..63 (RoPE frequencies of 64 interleaved pairs).
  2. Each cached key is reconstructed *before* RoPE as an additive sum of R key
     codewords per group of PPG pairs (layouts below).  A key codeword is the commutative 2x2 block
     [[a,-b],[b,a]]; applied to e_1 it gives the pair value (a, b).
     -- CommVQ review page (pith.science, arXiv 2506.18879), "key_machinery":
        per-subspace codebook matrices [[x, y], [-y, x]] that commute with the RoPE
        rotation R_m^i; group-shared indices; R residual rounds (additive).
  3. RoPE is applied as an explicit 2x2 rotation by angle theta_j * t at absolute
     position t.
  4. score_t = q . RoPE_t(k_t) / sqrt(128), q being the already-rotated query.
  5. Softmax with max subtraction; lse = m + ln(sum exp(s - m)).
  6. Each value is reconstructed as an additive sum of R codewords per group of VD
     dims (the CommVQ abstract on the aitopics.org "1-bit quantization" page: a value
     is recovered from its codes by a plain matrix product with the codebook), and
     out = sum_t w_t v_t.

Also here, each following the same pages:
  * qtable(): the query x key-codebook table P = conj(q_j) * c that the method
    precomputes once per query (CommVQ summary page, atlas.scime.ai, "Approach";
    review page "key_machinery").
  * score_from_table(): the score written in table form,
    sum_j Re(e^{i theta_j t} * sum_r P[G, r, code, p]) / sqrt(128).
  * value_bins() / output_from_bins(): the reordered value side, where softmax
    weights multiply the value codes before the codebook multiply (review page,
    "forward_implications", 4th item).
  * split_partials() / combine(): split-T partial softmax states and their
    log-sum-exp merge (standard flash-decode algebra; not on the pages).

Layouts (all row-major):
  q          [B, Hq, 128]                 pair j = dims (2j, 2j+1)
  key_cb     [Hkv, NG, R, NC, PPG, 2]      (group G, round r, code c, pair p, re/im)
  val_cb     [Hkv, NG, R, NC, VD]          (group G, round r, code c, dim d)
  key_codes  [B, Hkv, T_cap, R, NG] uint8  (token-major; attend() also takes the
  val_codes  [B, Hkv, T_cap, R, NG] uint8   planar order [B, Hkv, NG, R, T_cap])
  seq_lens   [B] int
Query head hq reads KV head hq // (Hq // Hkv).  A group G is PPG consecutive RoPE
pairs of the key (pairs PPG*G .. PPG*G + PPG - 1) and VD = 2*PPG consecutive dims of
the value (the review page, "key_machinery": neighbouring sub-vectors use the same
quantization index, g of them per group).  Two instances are used, read off the codebook shapes:
  g = 8 scalars:  NG = 16, PPG = 4,  NC = 256 codewords, R = 1 or 2 (1 or 2 bits);
  g = 64 scalars: NG = 2,  PPG = 32, NC = 64 codewords,  R = 11 or 21 -- the paper's own
                  parameterization, R log2(64) / 64 = 1.03 or 1.97 bits (CommVQ summary
                  page, "Key results" and "Limitations").
"""
from __future__ import annotations

import math

import numpy as np

HEAD_DIM = 128
N_PAIRS = 64
N_GROUPS = 16
PAIRS_PER_GROUP = 4
VDIMS_PER_GROUP = 8
N_CODES = 256
SCALE = 1.0 / math.sqrt(HEAD_DIM)


# ---------------------------------------------------------------------------
# step 1: RoPE frequencies
# ---------------------------------------------------------------------------
def rope_theta(base: float) -> np.ndarray:
    """theta_j = base^(-2j/128) for the 64 interleaved pairs, float64."""
    j = np.arange(N_PAIRS, dtype=np.float64)
    return np.power(np.float64(base), -2.0 * j / HEAD_DIM)


# ---------------------------------------------------------------------------
# step 2 / 6: additive codebook reconstruction
# ---------------------------------------------------------------------------
def decode_keys(key_cb_h: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """Pre-RoPE keys [T, 128] from codes [T, R, NG] and one head's codebook
    [NG, R, NC, PPG, 2].  Pair j = PPG*G + p holds sum_r key_cb[G, r, code[r, G], p]."""
    codes = np.asarray(codes)
    T, R, _ = codes.shape
    cb = np.asarray(key_cb_h, dtype=np.float64)
    n_groups, ppg = cb.shape[0], cb.shape[3]
    assert n_groups * ppg == N_PAIRS and codes.shape[2] == n_groups
    k = np.zeros((T, n_groups, ppg, 2), dtype=np.float64)
    for r in range(R):
        for g in range(n_groups):
            k[:, g] += cb[g, r][codes[:, r, g]]
    # [T, G, p, (re, im)] -> dim 2 PPG G + 2p + comp = 2j + comp with j = PPG G + p
    return k.reshape(T, HEAD_DIM)


def decode_values(val_cb_h: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """Values [T, 128] from codes [T, R, NG] and one head's codebook [NG, R, NC, VD].
    Dim VD*G + d holds sum_r val_cb[G, r, code[r, G], d]."""
    codes = np.asarray(codes)
    T, R, _ = codes.shape
    cb = np.asarray(val_cb_h, dtype=np.float64)
    n_groups, vd = cb.shape[0], cb.shape[3]
    assert n_groups * vd == HEAD_DIM and codes.shape[2] == n_groups
    v = np.zeros((T, n_groups, vd), dtype=np.float64)
    for r in range(R):
        for g in range(n_groups):
            v[:, g] += cb[g, r][codes[:, r, g]]
    return v.reshape(T, HEAD_DIM)


# ---------------------------------------------------------------------------
# step 3: RoPE as an explicit 2x2 rotation
# ---------------------------------------------------------------------------
def apply_rope(x: np.ndarray, positions: np.ndarray, theta: np.ndarray) -> np.ndarray:
    """Rotate each pair (x[2j], x[2j+1]) of x [T, 128] by the matrix
    [[cos a, -sin a], [sin a, cos a]] with a = theta_j * position."""
    ang = np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :]
    c = np.cos(ang)
    s = np.sin(ang)
    xe = x[:, 0::2]
    xo = x[:, 1::2]
    out = np.empty_like(x, dtype=np.float64)
    out[:, 0::2] = c * xe - s * xo
    out[:, 1::2] = s * xe + c * xo
    return out


def kv_head_of(hq: int, n_q_heads: int, n_kv_heads: int) -> int:
    return hq // (n_q_heads // n_kv_heads)


# ---------------------------------------------------------------------------
# steps 2-5: scores of one query head against one sequence
# ---------------------------------------------------------------------------
def scores(q_vec, key_cb_h, key_codes_bh, seq_len, base, chunk=32768):
    """Scaled scores s_t, t < seq_len, for one query vector [128] (float64)."""
    theta = rope_theta(base)
    q = np.asarray(q_vec, dtype=np.float64)
    out = np.empty(seq_len, dtype=np.float64)
    for t0 in range(0, seq_len, chunk):
        t1 = min(seq_len, t0 + chunk)
        k = decode_keys(key_cb_h, key_codes_bh[t0:t1])
        rk = apply_rope(k, np.arange(t0, t1), theta)
        out[t0:t1] = (rk @ q) * SCALE
    return out


def softmax_weights(s: np.ndarray):
    """Weights w_t = exp(s_t - m) / sum, plus lse = m + ln sum exp(s - m)."""
    if s.size == 0:
        return np.zeros(0), -math.inf
    m = float(np.max(s))
    e = np.exp(s - m)
    l = float(np.sum(e))
    return e / l, m + math.log(l)


def attend_head(q_vec, key_cb_h, val_cb_h, key_codes_bh, val_codes_bh, seq_len, base,
                chunk=32768):
    """(out [128], lse) for one query head: the plain definition, steps 1-6."""
    if seq_len == 0:
        return np.zeros(HEAD_DIM), -math.inf
    s = scores(q_vec, key_cb_h, key_codes_bh, seq_len, base, chunk)
    w, lse = softmax_weights(s)
    out = np.zeros(HEAD_DIM)
    for t0 in range(0, seq_len, chunk):
        t1 = min(seq_len, t0 + chunk)
        out += w[t0:t1] @ decode_values(val_cb_h, val_codes_bh[t0:t1])
    return out, lse


def token_major(codes):
    """Planar codes [B, Hkv, NG, R, T] viewed token-major [B, Hkv, T, R, NG] (a
    transposed view; no value changes)."""
    return np.transpose(np.asarray(codes), (0, 1, 4, 3, 2))


def attend(q, key_cb, val_cb, key_codes, val_codes, seq_lens, base, heads=None,
           codes_layout="token"):
    """Full decode step.  Returns out [B, Hq, 128] and lse [B, Hq] (float64).

    `heads`, if given, is an iterable of (b, hq) to compute; other entries are NaN.
    `codes_layout` "planar" takes codes as [B, Hkv, NG, R, T_cap]; "planar6" takes them
    packed 6 bits per code along the token axis (oracle/pack.py), [B, Hkv, NG, R, 3 T_cap/4].
    """
    if codes_layout == "planar6":
        from .pack import unpack_codes6
        n = key_codes.shape[-1] * 4 // 3
        key_codes, val_codes = unpack_codes6(key_codes, n), unpack_codes6(val_codes, n)
        codes_layout = "planar"
    if codes_layout == "planar":
        key_codes, val_codes = token_major(key_codes), token_major(val_codes)
    q = np.asarray(q, dtype=np.float64)
    B, Hq, _ = q.shape
    Hkv = key_codes.shape[1]
    out = np.full((B, Hq, HEAD_DIM), np.nan)
    lse = np.full((B, Hq), np.nan)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, hq in todo:
        h = kv_head_of(hq, Hq, Hkv)
        out[b, hq], lse[b, hq] = attend_head(
            q[b, hq], key_cb[h], val_cb[h], key_codes[b, h], val_codes[b, h],
            int(seq_lens[b]), base)
    return out, lse


# ---------------------------------------------------------------------------
# the method's precompute: query x key-codebook table
# ---------------------------------------------------------------------------
def qtable(q, key_cb, n_kv_heads):
    """P[b, hq, G, r, c, p, (re, im)] = conj(q_j) * c with q_j = q[2j] + i q[2j+1],
    c = a + i b the codeword of KV head hq // (Hq/Hkv), j = PPG*G + p."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, _ = q.shape
    cb = np.asarray(key_cb, dtype=np.float64)
    n_groups, R, n_codes, ppg = cb.shape[1], cb.shape[2], cb.shape[3], cb.shape[4]
    P = np.empty((B, Hq, n_groups, R, n_codes, ppg, 2))
    for b in range(B):
        for hq in range(Hq):
            h = kv_head_of(hq, Hq, n_kv_heads)
            qc = (q[b, hq, 0::2] - 1j * q[b, hq, 1::2]).reshape(n_groups, 1, 1, ppg)
            c = cb[h, ..., 0] + 1j * cb[h, ..., 1]          # [NG, R, NC, PPG]
            prod = qc * c
            P[b, hq, ..., 0] = prod.real
            P[b, hq, ..., 1] = prod.imag
    return P


def score_from_table(P_bh, key_codes_bh, seq_len, base):
    """score_t = sum_{G,p} Re(e^{i theta_{PPG G+p} t} * sum_r P[G, r, code_{t,r,G}, p]) / sqrt(128)."""
    theta = rope_theta(base)
    T = seq_len
    codes = key_codes_bh[:T]
    R = codes.shape[1]
    n_groups, ppg = P_bh.shape[0], P_bh.shape[3]
    z = np.zeros((T, n_groups, ppg), dtype=np.complex128)
    for r in range(R):
        for g in range(n_groups):
            ent = P_bh[g, r][codes[:, r, g]]               # [T, PPG, 2]
            z[:, g] += ent[..., 0] + 1j * ent[..., 1]
    phase = np.exp(1j * np.arange(T, dtype=np.float64)[:, None] * theta[None, :])
    return np.real(phase * z.reshape(T, N_PAIRS)).sum(axis=1) * SCALE


# ---------------------------------------------------------------------------
# the method's value reorder: probability bins times the value codebook
# ---------------------------------------------------------------------------
def value_bins(w, val_codes_bh, n_codes=N_CODES):
    """bins[G, r, c] = sum_t w_t [val_code_{t,r,G} == c]."""
    w = np.asarray(w, dtype=np.float64)
    T = w.shape[0]
    codes = val_codes_bh[:T]
    R, n_groups = codes.shape[1], codes.shape[2]
    bins = np.zeros((n_groups, R, n_codes))
    for r in range(R):
        for g in range(n_groups):
            np.add.at(bins[g, r], codes[:, r, g], w)
    return bins


def output_from_bins(bins, val_cb_h):
    """out[VD*G + d] = sum_{r, c} bins[G, r, c] * val_cb[G, r, c, d]."""
    cb = np.asarray(val_cb_h, dtype=np.float64)
    out = np.einsum("grc,grcd->gd", bins, cb)
    return out.reshape(HEAD_DIM)


# ---------------------------------------------------------------------------
# split-T partial states and their merge
# ---------------------------------------------------------------------------
def split_partials(s, v, bounds):
    """For token ranges bounds = [(t0, t1), ...] over scores s [T] and values v [T, 128]:
    m = max s, l = sum exp(s - m), o = sum exp(s - m) v.  Empty range: (-inf, 0, 0)."""
    ms, ls, os_ = [], [], []
    for t0, t1 in bounds:
        if t1 <= t0:
            ms.append(-math.inf)
            ls.append(0.0)
            os_.append(np.zeros(HEAD_DIM))
            continue
        m = float(np.max(s[t0:t1]))
        e = np.exp(s[t0:t1] - m)
        ms.append(m)
        ls.append(float(e.sum()))
        os_.append(e @ v[t0:t1])
    return np.array(ms), np.array(ls), np.array(os_)


def combine(m, l, o):
    """M = max m_s; L = sum l_s e^{m_s - M}; out = sum o_s e^{m_s - M} / L; lse = M + ln L.
    All splits empty -> out 0, lse -inf."""
    m = np.asarray(m, dtype=np.float64)
    if m.size == 0 or not np.isfinite(m).any():
        return np.zeros(HEAD_DIM), -math.inf
    M = float(np.max(m))
    f = np.where(np.isfinite(m), np.exp(m - M), 0.0)
    L = float(np.sum(np.asarray(l) * f))
    out = (np.asarray(o) * f[:, None]).sum(axis=0) / L
    return out, M + math.log(L)


# ---------------------------------------------------------------------------
# size accounting of the cache layout
# ---------------------------------------------------------------------------
def code_bytes_per_token(R: int, n_groups: int = N_GROUPS) -> int:
    """Bytes of key + value codes one token of one KV head occupies:
    one uint8 per (group, round), for keys and again for values."""
    return 2 * R * n_groups


def fp16_kv_bytes_per_token() -> int:
    """Bytes of the same token's key and value in FP16."""
    return 2 * HEAD_DIM * 2


def avg_bits(R: int, n_codes: int, group: int) -> float:
    """Average bits per quantized unit: R * log2(N_c') / g, the bit-rate formula of the
    review page's "key_machinery" (R residual rounds, N_c' codewords, group size g)."""
    return R * math.log2(n_codes) / group
