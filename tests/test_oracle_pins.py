"""Pins of the float64 oracle against things other than itself: a scalar brute force,
closed forms derived by hand, identities of the method (commutativity, table form,
value reorder, split merge), invariants of RoPE and figures the pages print.

Each test names the passage it follows.  The last block plants plausible mistakes
in the oracle (on the CPU) and checks that some pin catches each of them.
"""
import json
import math
import os

import numpy as np
import pytest

import workloads
from oracle import brute
from oracle import cvq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _case(T=6, R=1, Hq=2, Hkv=1, seed=0, cb_std=1.0, q_dtype="f32", codes="uniform"):
    return workloads.small(batch=1, n_q_heads=Hq, n_kv_heads=Hkv, t_cap=T, R=R,
                           q_dtype=q_dtype, cb_std=cb_std, codes=codes, seed=seed)


# ---------------------------------------------------------------------------
# 1. brute force on T <= 8
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("T,R,Hq,Hkv,seed", [(1, 1, 1, 1, 0), (3, 2, 2, 1, 1), (8, 1, 4, 2, 2),
                                             (8, 2, 4, 1, 3), (5, 2, 2, 2, 4)])
def test_brute_force_agrees(T, R, Hq, Hkv, seed):
    d = _case(T=T, R=R, Hq=Hq, Hkv=Hkv, seed=seed)
    out, lse = O.attend(d["q"], d["key_cb"], d["val_cb"], d["key_codes"], d["val_codes"],
                        d["seq_lens"], d["rope_base"])
    for hq in range(Hq):
        h = O.kv_head_of(hq, Hq, Hkv)
        bo, bl = brute.brute_attend_head(d["q"][0, hq].tolist(), d["key_cb"][h], d["val_cb"][h],
                                         d["key_codes"][0, h], d["val_codes"][0, h], T,
                                         d["rope_base"])
        np.testing.assert_allclose(out[0, hq], bo, rtol=0, atol=1e-12)
        assert abs(lse[0, hq] - bl) <= 1e-12


def test_brute_force_long_positions():
    """Scalar scores at large absolute positions (angles up to ~1.3e5 rad): eight keys
    placed at positions 131064..131071, compared score by score."""
    d = _case(T=8, R=1, Hq=1, seed=9)
    theta = O.rope_theta(d["rope_base"])
    q = d["q"][0, 0].astype(np.float64)
    k = O.decode_keys(d["key_cb"][0], d["key_codes"][0, 0])
    pos = np.arange(131064, 131072)
    s_or = (O.apply_rope(k, pos, theta) @ q) * O.SCALE
    for i, t in enumerate(pos):
        acc = 0.0
        for j in range(64):
            a = (d["rope_base"] ** (-2.0 * j / 128.0)) * int(t)
            x, y = k[i, 2 * j], k[i, 2 * j + 1]
            acc += q[2 * j] * (math.cos(a) * x - math.sin(a) * y) + q[2 * j + 1] * (
                math.sin(a) * x + math.cos(a) * y)
        assert abs(acc / math.sqrt(128) - s_or[i]) < 1e-11


# ---------------------------------------------------------------------------
# 2. commutativity of the codeword family with RoPE (review page, key_machinery)
# ---------------------------------------------------------------------------
def test_codeword_commutes_with_rope():
    rng = np.random.default_rng(0)
    for _ in range(200):
        a, b, ang = rng.standard_normal(3) * np.array([1, 1, 1e4])
        x = rng.standard_normal(2)
        C = np.array([[a, -b], [b, a]])
        Rm = np.array([[math.cos(ang), -math.sin(ang)], [math.sin(ang), math.cos(ang)]])
        np.testing.assert_allclose(Rm @ (C @ x), C @ (Rm @ x), atol=1e-13)
        # the pages write the family as [[x, y], [-y, x]]: the same set with y = -b
        Cp = np.array([[a, b], [-b, a]])
        np.testing.assert_allclose(Rm @ Cp, Cp @ Rm, atol=1e-13)


def test_rope_is_complex_multiplication():
    """apply_rope on pair j equals e^{i theta_j t} (x + i y) computed with numpy complex."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 128))
    pos = np.array([0, 1, 17, 4095, 131071])
    th = O.rope_theta(500000.0)
    got = O.apply_rope(x, pos, th)
    z = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(1j * pos[:, None] * th[None, :])
    np.testing.assert_allclose(got[:, 0::2], z.real, atol=1e-12)
    np.testing.assert_allclose(got[:, 1::2], z.imag, atol=1e-12)


def test_rope_relative_position():
    """<R_m q, R_t k> depends only on t - m (the property RoPE exists for)."""
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 128))
    k = rng.standard_normal((1, 128))
    th = O.rope_theta(500000.0)
    base = float((O.apply_rope(q, [3], th) @ O.apply_rope(k, [10], th).T)[0, 0])
    for shift in (1, 100, 9999):
        s = float((O.apply_rope(q, [3 + shift], th) @ O.apply_rope(k, [10 + shift], th).T)[0, 0])
        assert abs(s - base) < 1e-10


# ---------------------------------------------------------------------------
# closed forms derived by hand (sign of the rotation, pair layout, theta_j, GQA map)
# ---------------------------------------------------------------------------
def _onehot_case(R=1, Hq=1, Hkv=1, T=2):
    key_cb = np.zeros((Hkv, 16, R, 256, 4, 2), np.float32)
    val_cb = np.zeros((Hkv, 16, R, 256, 8), np.float32)
    key_codes = np.zeros((1, Hkv, T, R, 16), np.uint8)
    val_codes = np.zeros((1, Hkv, T, R, 16), np.uint8)
    q = np.zeros((1, Hq, 128), np.float32)
    return q, key_cb, val_cb, key_codes, val_codes


def test_closed_form_rotation_sign():
    """Key pair 0 = (1, 0) (codeword a=1, b=0), query pair 0 = (0, 1), theta_0 = 1:
    RoPE_t k = (cos t, sin t), so s_t = sin(t)/sqrt(128).  With values v_0 = 1, v_1 = 3
    in dim 0: out[0] = (1 + 3 e^{s_1}) / (1 + e^{s_1}), lse = ln(1 + e^{s_1})."""
    q, kc, vc, kcode, vcode = _onehot_case()
    kc[0, 0, 0, 0, 0] = (1.0, 0.0)
    q[0, 0, 1] = 1.0
    vc[0, 0, 0, 0, 0] = 1.0
    vc[0, 0, 0, 1, 0] = 3.0
    vcode[0, 0, 1, 0, 0] = 1
    out, lse = O.attend(q, kc, vc, kcode, vcode, np.array([2]), 500000.0)
    s1 = math.sin(1.0) / math.sqrt(128.0)
    assert abs(out[0, 0, 0] - (1 + 3 * math.exp(s1)) / (1 + math.exp(s1))) < 1e-14
    assert abs(lse[0, 0] - math.log(1 + math.exp(s1))) < 1e-14
    assert np.all(out[0, 0, 1:] == 0)


def test_closed_form_pair_and_theta():
    """Pair j = 5 lives in dims (10, 11), group 1, slot 1.  Codeword (a, b) = (2, -1)
    there, query pair (q10, q11) = (0.5, 0.25), token at t = 3:
    s = Re(conj(q) e^{i theta_5 3} (a + i b)) / sqrt(128), theta_5 = 500000^(-10/128)."""
    q, kc, vc, kcode, vcode = _onehot_case(T=4)
    kc[0, 1, 0, 7, 1] = (2.0, -1.0)
    kcode[0, 0, 3, 0, 1] = 7
    q[0, 0, 10], q[0, 0, 11] = 0.5, 0.25
    s = O.scores(q[0, 0], kc[0], kcode[0, 0], 4, 500000.0)
    th5 = 500000.0 ** (-10.0 / 128.0)
    z = complex(0.5, -0.25) * complex(math.cos(3 * th5), math.sin(3 * th5)) * complex(2.0, -1.0)
    assert abs(s[3] - z.real / math.sqrt(128.0)) < 1e-15
    assert np.all(s[:3] == 0)


def test_closed_form_residual_rounds_add():
    """R = 2: the key pair is the plain sum of the two rounds' codewords and the value
    dim the plain sum of the two rounds' entries (no per-round scale)."""
    q, kc, vc, kcode, vcode = _onehot_case(R=2, T=1)
    kc[0, 0, 0, 3, 0] = (1.0, 2.0)
    kc[0, 0, 1, 9, 0] = (0.5, -4.0)
    kcode[0, 0, 0, 0, 0] = 3
    kcode[0, 0, 0, 1, 0] = 9
    k = O.decode_keys(kc[0], kcode[0, 0])
    assert tuple(k[0, :2]) == (1.5, -2.0)
    vc[0, 15, 0, 4, 7] = 2.0
    vc[0, 15, 1, 200, 7] = 0.25
    vcode[0, 0, 0, 0, 15] = 4
    vcode[0, 0, 0, 1, 15] = 200
    v = O.decode_values(vc[0], vcode[0, 0])
    assert v[0, 127] == 2.25 and np.count_nonzero(v) == 1


def test_closed_form_gqa_mapping():
    """Hq = 8, Hkv = 2: query heads 0..3 read KV head 0, heads 4..7 read KV head 1."""
    assert [O.kv_head_of(h, 8, 2) for h in range(8)] == [0, 0, 0, 0, 1, 1, 1, 1]
    q, kc, vc, kcode, vcode = _onehot_case(Hq=8, Hkv=2, T=1)
    vc[1, 0, 0, 0, 0] = 5.0
    out, lse = O.attend(q, kc, vc, kcode, vcode, np.array([1]), 500000.0)
    assert np.all(out[0, :4, 0] == 0) and np.all(out[0, 4:, 0] == 5.0)
    assert np.all(lse == 0)


# ---------------------------------------------------------------------------
# 3-5. T = 1, equal scores, weights summing to one
# ---------------------------------------------------------------------------
def test_single_token_returns_its_value():
    d = _case(T=1, R=2, Hq=4, Hkv=1, seed=5)
    out, lse = O.attend(d["q"], d["key_cb"], d["val_cb"], d["key_codes"], d["val_codes"],
                        d["seq_lens"], d["rope_base"])
    v0 = O.decode_values(d["val_cb"][0], d["val_codes"][0, 0, :1])[0]
    for hq in range(4):
        assert np.array_equal(out[0, hq], v0)
        s0 = O.scores(d["q"][0, hq], d["key_cb"][0], d["key_codes"][0, 0], 1, d["rope_base"])[0]
        assert lse[0, hq] == s0


def test_equal_scores_give_mean():
    d = _case(T=257, R=1, Hq=1, seed=6)
    q0 = np.zeros_like(d["q"])
    out, lse = O.attend(q0, d["key_cb"], d["val_cb"], d["key_codes"], d["val_codes"],
                        d["seq_lens"], d["rope_base"])
    v = O.decode_values(d["val_cb"][0], d["val_codes"][0, 0])
    np.testing.assert_allclose(out[0, 0], v.mean(axis=0), rtol=0, atol=1e-13)
    assert abs(lse[0, 0] - math.log(257)) < 1e-13


def test_softmax_weights_sum_to_one():
    d = _case(T=4096, R=2, Hq=1, seed=7)
    s = O.scores(d["q"][0, 0], d["key_cb"][0], d["key_codes"][0, 0], 4096, d["rope_base"])
    w, lse = O.softmax_weights(s)
    assert abs(w.sum() - 1.0) < 1e-13
    assert abs(lse - math.log(np.exp(s).sum())) < 1e-12


def test_empty_sequence():
    d = _case(T=8, R=1, Hq=2)
    out, lse = O.attend(d["q"], d["key_cb"], d["val_cb"], d["key_codes"], d["val_codes"],
                        np.array([0]), d["rope_base"])
    assert np.all(out == 0) and np.all(np.isneginf(lse))


# ---------------------------------------------------------------------------
# 6. table form == reconstruct form (review page, key_machinery: precompute once)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("R", [1, 2])
def test_table_form_equals_reconstruct_form(R):
    d = _case(T=2000, R=R, Hq=4, Hkv=1, seed=10 + R)
    P = O.qtable(d["q"], d["key_cb"], 1)
    for hq in range(4):
        a = O.score_from_table(P[0, hq], d["key_codes"][0, 0], 2000, d["rope_base"])
        b = O.scores(d["q"][0, hq], d["key_cb"][0], d["key_codes"][0, 0], 2000, d["rope_base"])
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_qtable_entries_by_hand():
    """P = conj(q_j) c: q pair (3, 4) -> 3 - 4i; c = 1 + 2i -> (3 - 4i)(1 + 2i) = 11 + 2i."""
    q = np.zeros((1, 1, 128))
    q[0, 0, 2 * 6], q[0, 0, 2 * 6 + 1] = 3.0, 4.0          # pair 6 = group 1, slot 2
    kc = np.zeros((1, 16, 1, 256, 4, 2))
    kc[0, 1, 0, 42, 2] = (1.0, 2.0)
    P = O.qtable(q, kc, 1)
    assert tuple(P[0, 0, 1, 0, 42, 2]) == (11.0, 2.0)
    assert np.count_nonzero(P) == 2


# ---------------------------------------------------------------------------
# 7. reorder identity (review page, forward_implications: softmax weights multiply
#    the value codes before the codebook multiply)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("R,codes", [(1, "uniform"), (2, "zipf1.1")])
def test_value_reorder_identity(R, codes):
    d = _case(T=3000, R=R, Hq=1, seed=20 + R, codes=codes)
    s = O.scores(d["q"][0, 0], d["key_cb"][0], d["key_codes"][0, 0], 3000, d["rope_base"])
    w, _ = O.softmax_weights(s)
    direct = w @ O.decode_values(d["val_cb"][0], d["val_codes"][0, 0])
    bins = O.value_bins(w, d["val_codes"][0, 0])
    np.testing.assert_allclose(O.output_from_bins(bins, d["val_cb"][0]), direct, atol=1e-12)
    assert abs(bins.sum() - 16 * R) < 1e-12            # each (G, r) row sums to 1


# ---------------------------------------------------------------------------
# 8. split invariance of the partial-state merge
# ---------------------------------------------------------------------------
def test_split_invariance():
    d = _case(T=5000, R=2, Hq=1, seed=30)
    s = O.scores(d["q"][0, 0], d["key_cb"][0], d["key_codes"][0, 0], 5000, d["rope_base"])
    v = O.decode_values(d["val_cb"][0], d["val_codes"][0, 0])
    ref, ref_lse = O.attend_head(d["q"][0, 0], d["key_cb"][0], d["val_cb"][0],
                                 d["key_codes"][0, 0], d["val_codes"][0, 0], 5000,
                                 d["rope_base"])
    rng = np.random.default_rng(0)
    for n in (1, 2, 7, 33):
        cuts = np.sort(rng.integers(0, 5001, size=n - 1))
        edges = [0, *cuts.tolist(), 5000]
        bounds = list(zip(edges[:-1], edges[1:])) + [(5000, 5000)]   # plus an empty split
        m, l, o = O.split_partials(s, v, bounds)
        out, lse = O.combine(m, l, o)
        np.testing.assert_allclose(out, ref, atol=1e-13)
        assert abs(lse - ref_lse) < 1e-12


def test_combine_all_empty():
    out, lse = O.combine([-math.inf, -math.inf], [0.0, 0.0], np.zeros((2, 128)))
    assert np.all(out == 0) and math.isinf(lse) and lse < 0


# ---------------------------------------------------------------------------
# 9. figures the pages print: size reduction and bit rates
# ---------------------------------------------------------------------------
def _golden():
    with open(os.path.join(GOLDEN, "page_figures.json")) as f:
        return json.load(f)


def test_two_bit_size_reduction_matches_page():
    g = _golden()["two_bit_fp16_reduction_percent"]
    red = 100.0 * (1 - O.code_bytes_per_token(2) / O.fp16_kv_bytes_per_token())
    assert red == g["value"]
    # and the layout the generator draws is that size
    d = _case(T=10, R=2)
    assert d["key_codes"][0, 0, 0].nbytes + d["val_codes"][0, 0, 0].nbytes == O.code_bytes_per_token(2)


@pytest.mark.parametrize("key", ["commvq1_avg_bits", "commvq2_avg_bits", "table9_last_row_avg_bits"])
def test_avg_bits_match_page(key):
    g = _golden()[key]
    assert abs(O.avg_bits(g["R"], g["n_codes"], g["group"]) - g["value"]) <= g["tol"]


def test_instance_is_one_and_two_bits():
    """The instance's key group is 4 pairs = 8 scalars with 256 codewords: 1 bit per
    scalar per round; values likewise (8 dims, 256 codewords)."""
    assert O.avg_bits(1, 256, 8) == 1.0 and O.avg_bits(2, 256, 8) == 2.0


# ---------------------------------------------------------------------------
# 9. the paper's own parameterization: 64-entry codebooks over groups of 64 scalars
#    (32 consecutive RoPE pairs share one index), R = 11 / 21 (CommVQ summary page,
#    "Key results" and "Limitations"; review page "key_machinery")
# ---------------------------------------------------------------------------
def _wide_case(T=6, R=3, Hq=2, Hkv=1, seed=0):
    return workloads.small(batch=1, n_q_heads=Hq, n_kv_heads=Hkv, t_cap=T, R=R, seed=seed,
                           cb_std=math.sqrt(1.0 / R), group_dim=64)


@pytest.mark.parametrize("T,R,Hq,Hkv,seed", [(1, 1, 1, 1, 40), (5, 3, 2, 1, 41), (8, 11, 4, 2, 42),
                                             (3, 21, 2, 1, 43)])
def test_wide_brute_force_agrees(T, R, Hq, Hkv, seed):
    d = _wide_case(T=T, R=R, Hq=Hq, Hkv=Hkv, seed=seed)
    assert d["key_codes"].shape == (1, Hkv, 2, R, T) and int(d["key_codes"].max()) < 64
    out, lse = O.attend(d["q"], d["key_cb"], d["val_cb"], d["key_codes"], d["val_codes"],
                        d["seq_lens"], d["rope_base"], codes_layout="planar")
    for hq in range(Hq):
        h = O.kv_head_of(hq, Hq, Hkv)
        # planar [G, r, t] -> nested [t][r][G], by explicit loops
        kcodes = [[[int(d["key_codes"][0, h, G, r, t]) for G in range(2)] for r in range(R)]
                  for t in range(T)]
        vcodes = [[[int(d["val_codes"][0, h, G, r, t]) for G in range(2)] for r in range(R)]
                  for t in range(T)]
        bo, bl = brute.brute_attend_head(d["q"][0, hq].tolist(), d["key_cb"][h], d["val_cb"][h],
                                         kcodes, vcodes, T, d["rope_base"])
        np.testing.assert_allclose(out[0, hq], bo, rtol=0, atol=1e-12)
        assert abs(lse[0, hq] - bl) <= 1e-12


def test_wide_closed_form_groups_and_rounds():
    """Every code 5 (keys) / 7 (values); key codeword entry of group G, round r, pair slot
    p = (100 (G+1) + p + 1) (r + 1) (1, -1), so pair j = 32 G + p of the decoded key is
    (100 (G+1) + p + 1) R (R+1)/2 (1, -1); value entry (1000 G + d) 2^-r, so value dim
    64 G + d is (1000 G + d)(2 - 2^(1-R))."""
    R = 11
    kc = np.zeros((2, R, 64, 32, 2))
    vc = np.zeros((2, R, 64, 64))
    for G in range(2):
        for r in range(R):
            for p in range(32):
                kc[G, r, 5, p] = np.array([1.0, -1.0]) * (100 * (G + 1) + p + 1) * (r + 1)
            vc[G, r, 7] = (1000.0 * G + np.arange(64)) * 2.0 ** -r
    k = O.decode_keys(kc, np.full((1, R, 2), 5))
    v = O.decode_values(vc, np.full((1, R, 2), 7))
    for j in range(64):
        G, p = divmod(j, 32)
        e = (100 * (G + 1) + p + 1) * R * (R + 1) / 2
        assert k[0, 2 * j] == e and k[0, 2 * j + 1] == -e
    for dd in range(128):
        G, d = divmod(dd, 64)
        assert abs(v[0, dd] - (1000 * G + d) * (2 - 2.0 ** (1 - R))) < 1e-9


def test_wide_table_form_equals_reconstruct_form():
    d = _wide_case(T=700, R=11, Hq=4, Hkv=1, seed=44)
    kt = O.token_major(d["key_codes"])
    P = O.qtable(d["q"], d["key_cb"], 1)
    assert P.shape == (1, 4, 2, 11, 64, 32, 2)
    for hq in range(4):
        a = O.score_from_table(P[0, hq], kt[0, 0], 700, d["rope_base"])
        b = O.scores(d["q"][0, hq], d["key_cb"][0], kt[0, 0], 700, d["rope_base"])
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_wide_value_reorder_identity():
    d = _wide_case(T=900, R=21, Hq=1, seed=45)
    kt, vt = O.token_major(d["key_codes"]), O.token_major(d["val_codes"])
    s = O.scores(d["q"][0, 0], d["key_cb"][0], kt[0, 0], 900, d["rope_base"])
    w, _ = O.softmax_weights(s)
    direct = w @ O.decode_values(d["val_cb"][0], vt[0, 0])
    bins = O.value_bins(w, vt[0, 0], n_codes=64)
    assert bins.shape == (2, 21, 64)
    np.testing.assert_allclose(O.output_from_bins(bins, d["val_cb"][0]), direct, atol=1e-12)
    assert abs(bins.sum() - 2 * 21) < 1e-12


def test_wide_sizes():
    """R = 11 / 21 with 64 codewords over 64-scalar groups: R log2(64) / 64 bits per scalar
    (1.03 / 1.97); one uint8 per (group, round) is 2 R bytes per token for keys and again
    for values."""
    assert O.avg_bits(11, 64, 64) == 66 / 64 and O.avg_bits(21, 64, 64) == 126 / 64
    assert O.code_bytes_per_token(11, n_groups=2) == 44
    d = _wide_case(T=4, R=11)
    assert d["key_codes"][0, 0, :, :, 0].nbytes * 2 == O.code_bytes_per_token(11, n_groups=2)


# ---------------------------------------------------------------------------
# planted mistakes: each must make at least one pin above fail
# ---------------------------------------------------------------------------
def _pins_pass():
    try:
        test_brute_force_agrees(8, 2, 4, 1, 3)
        test_closed_form_rotation_sign()
        test_closed_form_pair_and_theta()
        test_closed_form_residual_rounds_add()
        test_table_form_equals_reconstruct_form(2)
        test_value_reorder_identity(2, "zipf1.1")
        test_rope_is_complex_multiplication()
        test_wide_brute_force_agrees(8, 11, 4, 2, 42)
        test_wide_closed_form_groups_and_rounds()
        test_wide_value_reorder_identity()
    except AssertionError:
        return False
    return True


def test_pins_pass_unmodified():
    assert _pins_pass()


def _bad_rope_sign(x, positions, theta):
    return O_apply_rope_orig(x, positions, -theta)


def _bad_theta(base):
    j = np.arange(64, dtype=np.float64)
    return np.power(np.float64(base), -j / 128.0)


def _bad_pairs(x, positions, theta):          # half-split pairs instead of interleaved
    ang = np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[:, :64], x[:, 64:]
    out = np.empty_like(x)
    out[:, :64] = c * a - s * b
    out[:, 64:] = s * a + c * b
    return out


def _bad_decode_keys(key_cb_h, codes):         # drops the last residual round
    return O_decode_keys_orig(key_cb_h, codes[:, :1]) if codes.shape[1] > 1 else O_decode_keys_orig(key_cb_h, codes)


def _bad_decode_values(val_cb_h, codes):       # transposed (G, d) inside the value
    v = O_decode_values_orig(val_cb_h, codes)
    return v.reshape(-1, 16, 8).transpose(0, 2, 1).reshape(-1, 128)


def _bad_decode_keys_strided(key_cb_h, codes):   # group G = pairs G, G + NG, ... (strided)
    k = O_decode_keys_orig(key_cb_h, codes)
    ng, ppg = key_cb_h.shape[0], key_cb_h.shape[3]
    return k.reshape(-1, ng, ppg, 2).transpose(0, 2, 1, 3).reshape(-1, 128)


def _bad_value_bins(w, val_codes_bh, n_codes=256):  # ignores every round after the first
    b = O_value_bins_orig(w, val_codes_bh, n_codes)
    b[:, 1:] = 0.0
    return b


O_apply_rope_orig = O.apply_rope
O_value_bins_orig = O.value_bins
O_decode_keys_orig = O.decode_keys
O_decode_values_orig = O.decode_values


@pytest.mark.parametrize("attr,bad", [("apply_rope", _bad_rope_sign), ("rope_theta", _bad_theta),
                                      ("apply_rope", _bad_pairs), ("decode_keys", _bad_decode_keys),
                                      ("decode_values", _bad_decode_values),
                                      ("decode_keys", _bad_decode_keys_strided),
                                      ("value_bins", _bad_value_bins)])
def test_planted_mistake_is_caught(monkeypatch, attr, bad):
    monkeypatch.setattr(O, attr, bad)
    assert not _pins_pass()
