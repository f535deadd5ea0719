"""The synthetic input recipe (no GPU): the seeded generators produce what the design states
-- Zipf(1.1) code frequencies, bf16 queries rounded to nearest even, ragged lengths in
[1024, 8192], codes in range for both layouts, codebook scale, and the same bits on every
call.  The generators hold none of the method's arithmetic; these checks only pin the
inputs both the oracle and the GPU path are fed."""
import math

import numpy as np

import workloads

W = workloads.WORKLOADS


def test_zipf_code_frequencies():
    k = np.arange(1, 257, dtype=np.float64)
    p = k ** -1.1
    p /= p.sum()
    assert 0.20 < p[0] < 0.21                     # code 0 carries ~21% of the tokens
    n = 1_000_000
    c = workloads.zipf_codes(np.random.default_rng(5), (n,))
    freq = np.bincount(c, minlength=256) / n
    for code in (0, 1, 2, 10, 100, 255):
        se = math.sqrt(p[code] * (1 - p[code]) / n)
        assert abs(freq[code] - p[code]) < 5 * se, (code, freq[code], p[code])


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 1.0 + 2.0 ** -9], np.float32)
    bits, back = workloads.bf16_round(x)
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties go to the even mantissa (1.0);
    # 1 + 3*2^-8 is halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even): rounds up
    assert list(bits) == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x3F80]
    assert back[2] == np.float32(1.0 + 2.0 ** -6)
    rng = np.random.default_rng(0)
    y = rng.standard_normal(10000).astype(np.float32)
    _, yb = workloads.bf16_round(y)
    assert np.all(np.abs(yb - y) <= np.abs(y) * 2.0 ** -8)   # half an ulp of an 8-bit mantissa


def test_ragged_lengths():
    w = W["llama8b_batch16_ragged_R2_zipf"]
    lens = workloads.make_seq_lens(w)
    assert lens.shape == (16,) and lens.dtype == np.int32
    assert lens.min() >= 1024 and lens.max() <= 8192
    assert len(set(lens.tolist())) > 8                      # really ragged
    assert np.array_equal(lens, workloads.make_seq_lens(w))  # seeded


def test_generate_shapes_ranges_and_scale():
    d = workloads.small(batch=2, n_q_heads=8, n_kv_heads=2, t_cap=512, R=2, seed=3,
                        cb_std=math.sqrt(0.5))
    assert d["key_codes"].shape == (2, 2, 512, 2, 16) and d["key_codes"].dtype == np.uint8
    assert d["key_cb"].shape == (2, 16, 2, 256, 4, 2) and d["val_cb"].shape == (2, 16, 2, 256, 8)
    assert abs(d["key_cb"].std() - math.sqrt(0.5)) < 0.01
    assert abs(d["key_codes"].mean() - 127.5) < 1.5        # uniform over 0..255
    dw = workloads.small(batch=1, n_q_heads=4, n_kv_heads=1, t_cap=256, R=11, seed=4,
                         cb_std=math.sqrt(1 / 11), group_dim=64)
    assert dw["key_codes"].shape == (1, 1, 2, 11, 256)      # planar [B, Hkv, 2, R, T]
    assert dw["key_codes"].max() < 64 and dw["val_codes"].max() < 64
    assert dw["key_cb"].shape == (1, 2, 11, 64, 32, 2) and dw["val_cb"].shape == (1, 2, 11, 64, 64)
    assert dw["codes_layout"] == "planar" and d["codes_layout"] == "token"


def test_generate_is_reproducible_and_layers_differ():
    w = W["llama8b_32layers_B4_T65536_R2"]
    a = workloads.generate(w, layer=3, t_cap=128, batch=1)
    b = workloads.generate(w, layer=3, t_cap=128, batch=1)
    c = workloads.generate(w, layer=4, t_cap=128, batch=1)
    for k in ("key_cb", "val_cb", "key_codes", "val_codes", "q_bits"):
        assert np.array_equal(a[k], b[k]), k
    assert not np.array_equal(a["key_cb"], c["key_cb"])      # distinct codebooks per layer
    assert a["q_dtype"] == "bf16" and a["q_bits"].dtype == np.uint16
