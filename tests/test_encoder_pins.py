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
