"""GPU parity of the paper's own parameterization: 64-entry codebooks over groups of 64
scalars (32 RoPE pairs share one index per round), R = 11 / 21 rounds, planar codes
[B, Hkv, 2, R, t_cap], 4 query heads per KV head (cvq_decode_attn_gqa with
group_dim = 64, then cvq_combine).

The bar is the same as for the default layout: max |out - oracle| <= 2e-3 and lse
relative error <= 1e-4 against the float64 oracle, element by element at small sizes
(several tiles, ragged tails, empty splits, both round-slice counts) and on sampled heads
at the full LLaMA-3.1-8B layer sizes.
"""
import math

import numpy as np
import pytest

import workloads
from oracle import cvq_oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import compressed_attention_cvq_b200 as cvq
    from gpu_util import assert_close, run_gpu, run_oracle, to_device


def _wide(T, R, lens, seed, batch=2, Hkv=2, q_dtype="f32"):
    return workloads.small(batch=batch, n_q_heads=4 * Hkv, n_kv_heads=Hkv, t_cap=T, R=R,
                           seq_lens=np.asarray(lens, np.int32), seed=seed, q_dtype=q_dtype,
                           cb_std=math.sqrt(1.0 / R), group_dim=64)


@pytest.mark.parametrize("R,T,lens,splits", [
    (1, 512, [512, 300], 2),          # one round: 2-CTA cluster, shortest R loop
    (3, 1024, [1024, 77], 3),         # ragged tail inside a 16-token chunk
    (11, 2048, [2048, 1500], 4),      # the paper's 1-bit setting, several tiles per split
    (11, 2048, [2048, 5], 8),         # the short sequence leaves 7 of 8 splits empty
    (12, 768, [700, 768], 2),         # 2 round slices of 6
    (21, 1536, [1536, 999], 3),       # the paper's 2-bit setting: 4-CTA cluster, 11 + 10
    (22, 512, [512, 513 - 256], 1),   # the largest R: 11 + 11
])
def test_wide_matches_oracle(R, T, lens, splits):
    d = _wide(T, R, lens, seed=60 + R)
    out, lse = run_gpu(d, n_splits=splits)
    ref_out, ref_lse = run_oracle(d)
    assert_close(out, lse, ref_out, ref_lse)


def test_wide_bf16_query_and_default_splits():
    d = _wide(4096, 11, [4096, 2500], seed=70, q_dtype="bf16")
    out, lse = run_gpu(d)
    ref_out, ref_lse = run_oracle(d)
    assert_close(out, lse, ref_out, ref_lse)


def test_wide_empty_and_shared_codebooks():
    """seq_len 0 -> out 0, lse -inf; codebooks shared by the KV heads (head stride 0)."""
    d = _wide(256, 11, [0, 256], seed=71)
    d["key_cb"] = d["key_cb"][:1].copy()
    d["val_cb"] = d["val_cb"][:1].copy()
    dd = to_device(d)
    dd["key_cb"], dd["val_cb"] = dd["key_cb"][0].contiguous(), dd["val_cb"][0].contiguous()
    out, lse = run_gpu(d, n_splits=2, dd=dd)
    ref_out, ref_lse = O.attend(d["q"], np.broadcast_to(d["key_cb"], (2,) + d["key_cb"].shape[1:]),
                                np.broadcast_to(d["val_cb"], (2,) + d["val_cb"].shape[1:]),
                                d["key_codes"], d["val_codes"], d["seq_lens"], d["rope_base"],
                                codes_layout="planar")
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    assert_close(out, lse, ref_out, ref_lse)


def test_wide_top_code_bits_ignored():
    """Only the low 6 bits of a code byte are read: setting the top 2 bits changes nothing
    beyond the run-to-run rounding of the shared-memory bin atomics (their order varies)."""
    d = _wide(512, 11, [512, 400], seed=72)
    base_out, base_lse = run_gpu(d, n_splits=2)
    hi = dict(d)
    rng = np.random.default_rng(72)
    hi["key_codes"] = d["key_codes"] | (rng.integers(0, 4, d["key_codes"].shape, dtype=np.uint8) << 6)
    hi["val_codes"] = d["val_codes"] | (rng.integers(0, 4, d["val_codes"].shape, dtype=np.uint8) << 6)
    out, lse = run_gpu(hi, n_splits=2)
    np.testing.assert_allclose(out, base_out, rtol=0, atol=1e-6)
    np.testing.assert_allclose(lse, base_lse, rtol=1e-7, atol=0)
    ref_out, ref_lse = run_oracle(d)
    assert_close(out, lse, ref_out, ref_lse)


def test_wide_partials_invariants():
    """Per split: m is within 8 ln 2 below the split's true max; m + ln l and o / l match
    the oracle's split partials."""
    d = _wide(1024, 11, [1024, 600], seed=73)
    dd = to_device(d)
    shape = cvq.shape_of(dd["q"], dd["key_codes"], d["rope_base"], 64)
    S = 3
    po, pm, pl = cvq.decode_attn_gqa(shape, dd["q"], dd["key_cb"], dd["key_codes"],
                                     dd["val_codes"], dd["seq_lens"], dd["val_cb"], S)
    torch.cuda.synchronize()
    po, pm, pl = (x.cpu().numpy().astype(np.float64) for x in (po, pm, pl))
    C = cvq.split_tokens(shape, S)
    kt, vt = O.token_major(d["key_codes"]), O.token_major(d["val_codes"])
    for b in range(2):
        L = int(d["seq_lens"][b])
        for hq in range(8):
            h = hq // 4
            s = O.scores(d["q"][b, hq], d["key_cb"][h], kt[b, h], L, d["rope_base"])
            v = O.decode_values(d["val_cb"][h], vt[b, h, :L])
            bounds = [(i * C, min((i + 1) * C, L)) for i in range(S)]
            m, l, o = O.split_partials(s, v, bounds)
            for i in range(S):
                if not np.isfinite(m[i]):
                    assert np.isneginf(pm[b, hq, i]) and pl[b, hq, i] == 0
                    continue
                tol = 1e-4 * max(1.0, abs(m[i]))
                assert m[i] - 8 * math.log(2) - tol <= pm[b, hq, i] <= m[i] + tol
                lse_ref = m[i] + math.log(l[i])
                assert abs(pm[b, hq, i] + math.log(pl[b, hq, i]) - lse_ref) <= 1e-4 * max(1, abs(lse_ref))
                np.testing.assert_allclose(po[b, hq, i] / pl[b, hq, i], o[i] / l[i], atol=2e-3)


def test_wide_static_entry():
    d = _wide(1024, 11, [1024, 333], seed=74)
    dd = to_device(d)
    shape = cvq.shape_of(dd["q"], dd["key_codes"], d["rope_base"], 64)
    from compressed_attention_cvq_b200 import _binding as _b
    import ctypes
    out = torch.empty((2, 8, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((2, 8), dtype=torch.float32, device="cuda")
    st = _b.lib.cvq_attend_static(ctypes.byref(shape), dd["q"].data_ptr(), 0, dd["key_cb"].data_ptr(),
                                  8192 * 11, dd["key_codes"].data_ptr(), dd["val_codes"].data_ptr(),
                                  dd["seq_lens"].data_ptr(), dd["val_cb"].data_ptr(), 8192 * 11, 4,
                                  out.data_ptr(), lse.data_ptr(), None)
    assert st == 0
    torch.cuda.synchronize()
    ref_out, ref_lse = run_oracle(d)
    assert_close(out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
                 ref_out, ref_lse)


def test_wide_table_form_fails_loudly():
    d = _wide(256, 11, [256, 256], seed=75)
    dd = to_device(d)
    with pytest.raises(cvq.CvqError):
        run_gpu(d, form="table", dd=dd)


@pytest.mark.parametrize("R", [3, 11, 21])
def test_wide_naive_dequant_matches_oracle(R):
    """The naive comparison path in the paper's layout: every cached key (rotated by RoPE)
    and value decoded into fp16 equals the oracle's reconstruction to fp16 rounding."""
    lens = np.array([200, 77], np.int32)
    d = _wide(208, R, lens, seed=76 + R)
    dd = to_device(d)
    shape = cvq.shape_of(dd["q"], dd["key_codes"], d["rope_base"], 64)
    k, v = cvq.naive_dequant(shape, dd["key_cb"], dd["val_cb"], dd["key_codes"], dd["val_codes"],
                             dd["seq_lens"])
    torch.cuda.synchronize()
    k, v = k.float().cpu().numpy(), v.float().cpu().numpy()
    theta = O.rope_theta(d["rope_base"])
    kt, vt = O.token_major(d["key_codes"]), O.token_major(d["val_codes"])
    for b in range(2):
        for h in range(2):
            L = int(lens[b])
            rk = O.apply_rope(O.decode_keys(d["key_cb"][h], kt[b, h, :L]), np.arange(L), theta)
            vv = O.decode_values(d["val_cb"][h], vt[b, h, :L])
            np.testing.assert_allclose(k[b, h, :L], rk, rtol=2 ** -10, atol=1e-5)
            np.testing.assert_allclose(v[b, h, :L], vv, rtol=2 ** -10, atol=1e-6)
            assert np.all(k[b, h, L:] == 0) and np.all(v[b, h, L:] == 0)


@pytest.mark.parametrize("R,T", [(11, 1024), (21, 512)])
def test_wide_naive_attention_matches_oracle(R, T):
    d = _wide(T, R, [T, T // 3 + 5], seed=78 + R)
    out, lse = run_gpu(d, form="naive", n_splits=3)
    ref_out, ref_lse = run_oracle(d)
    assert_close(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("name,k", [("llama8b_layer_T131072_R11_g64", 3),
                                    ("llama8b_layer_T32768_R21_g64", 4)])
def test_wide_full_size(name, k):
    """The full layer in the launch configuration the benchmark times (default splits),
    checked on sampled query heads."""
    w = workloads.WORKLOADS[name]
    d = workloads.generate(w)
    out, lse = run_gpu(d)
    rng = np.random.default_rng(2)
    heads = [(0, int(h)) for h in rng.choice(w.n_q_heads, size=k, replace=False)]
    ref_out, ref_lse = run_oracle(d, heads=heads)
    assert_close(out, lse, ref_out, ref_lse, heads=heads)
