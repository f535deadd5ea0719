"""GPU checks of the packed 6-bit code layout of the paper's parameterization (64-entry
codebooks over 64-scalar groups; code_bits = 6: 4 codes in 3 bytes per planar row):

- cvq_pack_codes6 against the oracle's packer (oracle/pack.py), bit for bit, including
  input bytes whose top two bits are set (they are not part of a code);
- the decode (fused and split forms, and the naive comparison path) on packed codes
  against the float64 oracle on the same codes, at small sizes (ragged tails, empty
  splits, one and two round slices) and on sampled heads of the full 128K-token layer
  with R = 11 (the paper's 1-bit setting);
- the write side on packed rows: codes bit-exact against the oracle encoder followed by
  the oracle packer, neighbouring codes untouched, then attend on the appended cache.
"""
import math

import numpy as np
import pytest

import workloads
from oracle import encode as E
from oracle import pack as P

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import compressed_attention_cvq_b200 as cvq
    from gpu_util import assert_close, run_oracle, to_device


def _wide(T, R, lens, seed, batch=2, Hkv=2):
    return workloads.small(batch=batch, n_q_heads=4 * Hkv, n_kv_heads=Hkv, t_cap=T, R=R,
                           seq_lens=np.asarray(lens, np.int32), seed=seed,
                           cb_std=math.sqrt(1.0 / R), group_dim=64)


def _packed_on_device(d, dd):
    """The case's codes packed on the device, checked bit for bit against the oracle."""
    shape = cvq.shape_of(dd["q"], dd["key_codes"], d["rope_base"], 64)
    shape.code_bits = 6
    pk = cvq.pack_codes6(shape, dd["key_codes"])
    pv = cvq.pack_codes6(shape, dd["val_codes"])
    torch.cuda.synchronize()
    assert np.array_equal(pk.cpu().numpy(), P.pack_codes6(d["key_codes"]))
    assert np.array_equal(pv.cpu().numpy(), P.pack_codes6(d["val_codes"]))
    return pk, pv


def test_pack_matches_oracle_with_top_bits_set():
    d = _wide(128, 3, [128, 128], seed=90)
    rng = np.random.default_rng(90)
    d["key_codes"] = d["key_codes"] | (rng.integers(0, 4, d["key_codes"].shape, dtype=np.uint8) << 6)
    dd = to_device(d)
    _packed_on_device(d, dd)


@pytest.mark.parametrize("R,T,lens,splits,form", [
    (1, 512, [512, 300], 2, "gqa"),
    (11, 2048, [2048, 1500], 4, "gqa"),         # several tiles per split
    (11, 2048, [2048, 5], 8, "gqa_split"),      # 7 of 8 splits empty for the short sequence
    (11, 1024, [1000, 77], 3, "gqa"),           # ragged tails inside a packed 16-byte chunk
    (21, 1536, [1536, 999], 3, "gqa"),          # 2 round slices (11 + 10)
    (11, 512, [512, 333], 2, "naive"),          # the comparison path reads packed rows too
])
def test_packed_decode_matches_oracle(R, T, lens, splits, form):
    d = _wide(T, R, lens, seed=91 + R + splits)
    dd = to_device(d)
    pk, pv = _packed_on_device(d, dd)
    out, lse = cvq.attend(dd["q"], dd["key_cb"], dd["val_cb"], pk, pv, dd["seq_lens"],
                          d["rope_base"], n_splits=splits, form=form, code_bits=6)
    torch.cuda.synchronize()
    ref_out, ref_lse = run_oracle(d)
    assert_close(out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
                 ref_out, ref_lse)


def test_packed_full_size_128k_r11():
    """The paper's 1-bit setting at the full 128K-token layer, packed (1.03 bits per scalar
    stored), in the benchmark's split configuration, on sampled heads."""
    w = workloads.WORKLOADS["llama8b_layer_T131072_R11_g64"]
    d = workloads.generate(w)
    dd = to_device(d)
    shape = cvq.shape_of(dd["q"], dd["key_codes"], d["rope_base"], 64)
    shape.code_bits = 6
    pk = cvq.pack_codes6(shape, dd["key_codes"])
    pv = cvq.pack_codes6(shape, dd["val_codes"])
    assert pk.numel() == dd["key_codes"].numel() * 3 // 4
    out, lse = cvq.attend(dd["q"], dd["key_cb"], dd["val_cb"], pk, pv, dd["seq_lens"],
                          d["rope_base"], code_bits=6)
    torch.cuda.synchronize()
    heads = [(0, 2), (0, 19)]
    ref_out, ref_lse = run_oracle(d, heads=heads)
    assert_close(out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
                 ref_out, ref_lse, heads=heads)
    assert cvq.fault_status(clear=True) == 0


@pytest.mark.parametrize("R", [1, 11, 21])
def test_packed_append_bit_exact(R):
    d = _wide(64, R, [64, 64, 64], seed=95 + R, batch=3)
    rng = np.random.default_rng(950 + R)
    keys = rng.standard_normal((3, 2, 128), dtype=np.float32)
    vals = rng.standard_normal((3, 2, 128), dtype=np.float32)
    # positions 0, 5 and 63 sit at each of the three ways a 6-bit code meets byte edges
    positions = np.array([0, 5, 63], np.int32)
    dd = to_device(d)
    shape = cvq.shape_of(dd["q"], dd["key_codes"], d["rope_base"], 64)
    shape.code_bits = 6
    pk, pv = _packed_on_device(d, dd)
    cvq.encode_append(shape, torch.from_numpy(keys).cuda(), torch.from_numpy(vals).cuda(),
                      dd["key_cb"], dd["val_cb"], torch.from_numpy(positions).cuda(), pk, pv)
    kc, vc = d["key_codes"].copy(), d["val_codes"].copy()
    E.encode_append(keys, vals, d["key_cb"], d["val_cb"], positions, kc, vc, codes_layout="planar")
    torch.cuda.synchronize()
    assert np.array_equal(pk.cpu().numpy(), P.pack_codes6(kc))
    assert np.array_equal(pv.cpu().numpy(), P.pack_codes6(vc))


def test_packed_append_then_attend():
    d = _wide(512, 11, [300, 511], seed=99)
    rng = np.random.default_rng(99)
    keys = rng.standard_normal((2, 2, 128), dtype=np.float32)
    vals = rng.standard_normal((2, 2, 128), dtype=np.float32)
    dd = to_device(d)
    shape = cvq.shape_of(dd["q"], dd["key_codes"], d["rope_base"], 64)
    shape.code_bits = 6
    pk, pv = _packed_on_device(d, dd)
    cvq.encode_append(shape, torch.from_numpy(keys).cuda(), torch.from_numpy(vals).cuda(),
                      dd["key_cb"], dd["val_cb"], dd["seq_lens"].clone(), pk, pv)
    kc, vc = d["key_codes"].copy(), d["val_codes"].copy()
    E.encode_append(keys, vals, d["key_cb"], d["val_cb"], d["seq_lens"], kc, vc,
                    codes_layout="planar")
    d2 = dict(d, key_codes=kc, val_codes=vc, seq_lens=d["seq_lens"] + 1)
    out, lse = cvq.attend(dd["q"], dd["key_cb"], dd["val_cb"], pk, pv, dd["seq_lens"] + 1,
                          d["rope_base"], n_splits=2, code_bits=6)
    torch.cuda.synchronize()
    ref_out, ref_lse = run_oracle(d2)
    assert_close(out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
                 ref_out, ref_lse)
