"""Pins of the oracle's greedy residual encoder (the write side that appends a decode
step's key / value to the code cache).

- exact recovery: a vector that is itself a sum of codewords is encoded back to those
  codes (R = 1; and R = 2 when the second round's codewords are much smaller);
- optimality: each round's code is the nearest codeword to the residual (float64 check);
- keys round-trip through the decode oracle: decode_keys(encode(k)) reproduces k;
- positions outside the buffer are skipped; a planted arg-max is caught.
"""
import numpy as np
import pytest

from oracle import cvq_oracle as O
from oracle import encode as E


def _cb(rng, R, scale=(1.0, 1e-3), key=True):
    shape = (2, 16, R, 256, 4, 2) if key else (2, 16, R, 256, 8)
    cb = rng.standard_normal(shape).astype(np.float32)
    for r in range(R):
        cb[:, :, r] *= np.float32(scale[r])
    return cb


@pytest.mark.parametrize("R", [1, 2])
def test_exact_recovery_of_codeword_sums(R):
    rng = np.random.default_rng(R)
    kcb, vcb = _cb(rng, R), _cb(rng, R, key=False)
    codes = rng.integers(0, 256, size=(R, 16)).astype(np.uint8)
    k = O.decode_keys(kcb[1], codes[None])[0].astype(np.float32)
    v = O.decode_values(vcb[1], codes[None])[0].astype(np.float32)
    assert np.array_equal(E.encode_vector(k, kcb[1]), codes)
    assert np.array_equal(E.encode_vector(v, vcb[1]), codes)


def test_each_round_picks_the_nearest_codeword():
    rng = np.random.default_rng(7)
    cb = rng.standard_normal((2, 256, 8)).astype(np.float32)
    for _ in range(50):
        x = (rng.standard_normal(8) * 2).astype(np.float32)
        codes, _ = E.encode_group(x, cb)
        res = x.astype(np.float64)
        for r, c in enumerate(codes):
            d = ((res[None, :] - cb[r].astype(np.float64)) ** 2).sum(axis=1)
            assert d[c] <= d.min() + 1e-5 * (1 + d.min())
            res = res - cb[r, c]


def test_encoded_key_decodes_close_to_input():
    """With codebooks that tile the space finely (R = 2), decode(encode(k)) is close to k
    and closer than with R = 1 on the same first-round codebook."""
    rng = np.random.default_rng(3)
    kcb = _cb(rng, 2, scale=(1.0, 0.3))
    k = rng.standard_normal(128).astype(np.float32)
    c2 = E.encode_vector(k, kcb[0])
    err2 = np.linalg.norm(O.decode_keys(kcb[0], c2[None])[0] - k)
    c1 = E.encode_vector(k, kcb[0][:, :1])
    err1 = np.linalg.norm(O.decode_keys(kcb[0][:, :1], c1[None])[0] - k)
    assert err2 < err1 < np.linalg.norm(k)


def test_append_writes_only_the_given_positions():
    rng = np.random.default_rng(4)
    kcb, vcb = _cb(rng, 1), _cb(rng, 1, key=False)
    keys = rng.standard_normal((3, 2, 128)).astype(np.float32)
    vals = rng.standard_normal((3, 2, 128)).astype(np.float32)
    kc = np.full((3, 2, 10, 1, 16), 7, np.uint8)
    vc = np.full((3, 2, 10, 1, 16), 7, np.uint8)
    E.encode_append(keys, vals, kcb, vcb, np.array([0, 9, 10]), kc, vc)
    assert np.array_equal(kc[0, 1, 0], E.encode_vector(keys[0, 1], kcb[1]))
    assert np.array_equal(vc[1, 0, 9], E.encode_vector(vals[1, 0], vcb[0]))
    assert np.all(kc[2] == 7) and np.all(vc[2] == 7)          # position 10 >= T_cap: skipped
    assert np.all(kc[0, :, 1:] == 7) and np.all(kc[1, :, :9] == 7)


def test_planted_argmax_is_caught(monkeypatch):
    orig = E._dist32
    monkeypatch.setattr(E, "_dist32", lambda x, c: -orig(x, c))
    with pytest.raises(AssertionError):
        test_exact_recovery_of_codeword_sums(1)


# ---------------------------------------------------------------------------
# the paper's layout: 2 groups of 64 scalars, 64 codewords per (group, round)
# ---------------------------------------------------------------------------
def _wide_cb(rng, R, scales, key=True):
    shape = (2, 2, R, 64, 32, 2) if key else (2, 2, R, 64, 64)
    cb = rng.standard_normal(shape).astype(np.float32)
    for r in range(R):
        cb[:, :, r] *= np.float32(scales[r])
    return cb


def test_wide_exact_recovery_of_codeword_sums():
    """Codeword sums with rounds of decreasing scale (1, 1e-3, 1e-6) encode back to their
    codes: each round's nearest codeword is the one that was added."""
    rng = np.random.default_rng(11)
    R = 3
    kcb, vcb = _wide_cb(rng, R, (1.0, 1e-3, 1e-6)), _wide_cb(rng, R, (1.0, 1e-3, 1e-6), key=False)
    codes = rng.integers(0, 64, size=(R, 2)).astype(np.uint8)
    k = O.decode_keys(kcb[0], codes[None])[0].astype(np.float32)
    v = O.decode_values(vcb[1], codes[None])[0].astype(np.float32)
    assert np.array_equal(E.encode_vector(k, kcb[0]), codes)
    assert np.array_equal(E.encode_vector(v, vcb[1]), codes)


def test_wide_each_round_picks_the_nearest_codeword():
    rng = np.random.default_rng(12)
    cb = rng.standard_normal((11, 64, 64)).astype(np.float32) * np.float32(0.3)
    for _ in range(20):
        x = rng.standard_normal(64).astype(np.float32)
        codes, _ = E.encode_group(x, cb)
        res = x.astype(np.float64)
        for r, c in enumerate(codes):
            d = ((res[None, :] - cb[r].astype(np.float64)) ** 2).sum(axis=1)
            assert d[c] <= d.min() + 1e-5 * (1 + d.min())
            res = res - cb[r, c]


def test_wide_append_planar_positions():
    rng = np.random.default_rng(13)
    kcb, vcb = _wide_cb(rng, 2, (1.0, 0.3)), _wide_cb(rng, 2, (1.0, 0.3), key=False)
    keys = rng.standard_normal((2, 2, 128)).astype(np.float32)
    vals = rng.standard_normal((2, 2, 128)).astype(np.float32)
    kc = np.full((2, 2, 2, 2, 16), 99, np.uint8)        # [B, Hkv, NG, R, T_cap]
    vc = np.full((2, 2, 2, 2, 16), 99, np.uint8)
    E.encode_append(keys, vals, kcb, vcb, np.array([5, 16]), kc, vc, codes_layout="planar")
    assert np.array_equal(kc[0, 1, :, :, 5], E.encode_vector(keys[0, 1], kcb[1]).T)
    assert np.array_equal(vc[0, 0, :, :, 5], E.encode_vector(vals[0, 0], vcb[0]).T)
    assert np.all(kc[1] == 99) and np.all(vc[1] == 99)   # position 16 >= T_cap: skipped
    assert np.all(kc[0, :, :, :, :5] == 99) and np.all(kc[0, :, :, :, 6:] == 99)
    assert int(kc[0, :, :, :, 5].max()) < 64
