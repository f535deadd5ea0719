"""GPU parity of the write side (cvq_encode_append): greedy residual encoding of one new
key / value per (sequence, KV head) into the code cache.

A code is an integer decided by floating point, so both sides decide in the same
precision and order (fp32, dims summed 0..7, no fused multiply-add, ties to the smaller
code) and the codes must be bit-exact with the oracle's.  Bytes the call must not write
(other positions, sequences whose position is out of range) must be unchanged.
"""
import math

import numpy as np
import pytest

import workloads
from oracle import cvq_oracle as O
from oracle import encode as E

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import compressed_attention_cvq_b200 as cvq
    from gpu_util import assert_close, run_gpu, run_oracle, to_device

FILL = 0xA5


def _new_vectors(rng, d, near_codebook):
    """Keys / values [B, Hkv, 128] fp32 for one decode step: Gaussian, or a codeword sum
    plus small noise (what a trained encoder's inputs look like to its codebook)."""
    B, Hkv, R = d["batch"], d["n_kv_heads"], d["R"]
    if not near_codebook:
        return (rng.standard_normal((B, Hkv, 128), dtype=np.float32),
                rng.standard_normal((B, Hkv, 128), dtype=np.float32))
    codes = rng.integers(0, 256, size=(B, Hkv, 1, R, 16)).astype(np.uint8)
    k = np.stack([np.stack([O.decode_keys(d["key_cb"][h], codes[b, h])[0] for h in range(Hkv)])
                  for b in range(B)])
    v = np.stack([np.stack([O.decode_values(d["val_cb"][h], codes[b, h])[0] for h in range(Hkv)])
                  for b in range(B)])
    k = k + 0.05 * rng.standard_normal(k.shape)
    v = v + 0.05 * rng.standard_normal(v.shape)
    return k.astype(np.float32), v.astype(np.float32)


def _run(d, keys, vals, positions, key_cb=None, val_cb=None):
    key_cb = d["key_cb"] if key_cb is None else key_cb
    val_cb = d["val_cb"] if val_cb is None else val_cb
    kc = np.full(d["key_codes"].shape, FILL, np.uint8)
    vc = np.full(d["val_codes"].shape, FILL, np.uint8)
    dev = dict(keys=torch.from_numpy(keys).cuda(), vals=torch.from_numpy(vals).cuda(),
               kcb=torch.from_numpy(np.ascontiguousarray(key_cb)).cuda(),
               vcb=torch.from_numpy(np.ascontiguousarray(val_cb)).cuda(),
               pos=torch.from_numpy(np.asarray(positions, np.int32)).cuda(),
               kc=torch.from_numpy(kc.copy()).cuda(), vc=torch.from_numpy(vc.copy()).cuda())
    shape = cvq.make_shape(d["batch"], d["n_q_heads"], d["n_kv_heads"], d["R"], d["t_cap"],
                           d["rope_base"])
    cvq.encode_append(shape, dev["keys"], dev["vals"], dev["kcb"], dev["vcb"], dev["pos"],
                      dev["kc"], dev["vc"])
    torch.cuda.synchronize()
    # the oracle works on per-head codebooks; a shared one is the same array for every head
    Hkv = d["n_kv_heads"]
    kcb_h = key_cb if key_cb.ndim == 6 else np.broadcast_to(key_cb, (Hkv,) + key_cb.shape)
    vcb_h = val_cb if val_cb.ndim == 5 else np.broadcast_to(val_cb, (Hkv,) + val_cb.shape)
    E.encode_append(keys, vals, kcb_h, vcb_h, positions, kc, vc)
    return dev["kc"].cpu().numpy(), dev["vc"].cpu().numpy(), kc, vc


@pytest.mark.parametrize("R,near", [(1, False), (1, True), (2, False), (2, True)])
def test_codes_bit_exact(R, near):
    d = workloads.small(batch=3, n_q_heads=16, n_kv_heads=4, t_cap=37, R=R, seed=70 + R,
                        cb_std=math.sqrt(1.0 / R))
    rng = np.random.default_rng(700 + R + 10 * near)
    keys, vals = _new_vectors(rng, d, near)
    positions = np.array([0, 36, 17], np.int32)
    gk, gv, ok, ov = _run(d, keys, vals, positions)
    assert np.array_equal(gk, ok) and np.array_equal(gv, ov)
    # only [b, :, positions[b]] changed
    mask = np.ones(gk.shape, bool)
    for b, p in enumerate(positions):
        mask[b, :, p] = False
    assert np.all(gk[mask] == FILL) and np.all(gv[mask] == FILL)


def test_out_of_range_positions_write_nothing():
    d = workloads.small(batch=4, n_q_heads=8, n_kv_heads=2, t_cap=16, R=2, seed=72)
    rng = np.random.default_rng(72)
    keys, vals = _new_vectors(rng, d, False)
    positions = np.array([-1, 16, 1 << 30, 3], np.int32)
    gk, gv, ok, ov = _run(d, keys, vals, positions)
    assert np.array_equal(gk, ok) and np.array_equal(gv, ov)
    assert np.all(gk[:3] == FILL) and np.all(gv[:3] == FILL)
    assert not np.all(gk[3, :, 3] == FILL)


def test_shared_codebooks_and_ties():
    """Shared codebooks (head stride 0); codeword 200 duplicated from codeword 5 and the
    input equal to it, so both have distance 0 and the smaller code must win."""
    d = workloads.small(batch=2, n_q_heads=8, n_kv_heads=2, t_cap=8, R=1, seed=73)
    kcb = d["key_cb"][0].copy()
    vcb = d["val_cb"][0].copy()
    kcb[:, 0, 200] = kcb[:, 0, 5]
    vcb[:, 0, 200] = vcb[:, 0, 5]
    codes = np.full((1, 1, 16), 5, np.uint8)
    keys = np.broadcast_to(O.decode_keys(kcb, codes)[0].astype(np.float32), (2, 2, 128)).copy()
    vals = np.broadcast_to(O.decode_values(vcb, codes)[0].astype(np.float32), (2, 2, 128)).copy()
    gk, gv, ok, ov = _run(d, keys, vals, np.array([2, 7], np.int32), key_cb=kcb, val_cb=vcb)
    assert np.array_equal(gk, ok) and np.array_equal(gv, ov)
    assert np.all(gk[0, :, 2] == 5) and np.all(gv[1, :, 7] == 5)


def test_append_then_attend_matches_oracle():
    """One decode step end to end: encode the new token into the cache at seq_len, advance
    seq_len, attend over the cache; the result matches the oracle on the same codes."""
    d = workloads.small(batch=2, n_q_heads=8, n_kv_heads=2, t_cap=600, R=2, seed=74,
                        seq_lens=np.array([511, 200], np.int32), cb_std=math.sqrt(0.5))
    rng = np.random.default_rng(74)
    keys, vals = _new_vectors(rng, d, True)
    dd = to_device(d)
    shape = cvq.shape_of(dd["q"], dd["key_codes"], d["rope_base"])
    pos = dd["seq_lens"].clone()
    cvq.encode_append(shape, torch.from_numpy(keys).cuda(), torch.from_numpy(vals).cuda(),
                      dd["key_cb"], dd["val_cb"], pos, dd["key_codes"], dd["val_codes"])
    dd["seq_lens"] += 1
    kc, vc = d["key_codes"].copy(), d["val_codes"].copy()
    E.encode_append(keys, vals, d["key_cb"], d["val_cb"], d["seq_lens"], kc, vc)
    d2 = dict(d, key_codes=kc, val_codes=vc, seq_lens=d["seq_lens"] + 1)
    assert np.array_equal(dd["key_codes"].cpu().numpy(), kc)
    assert np.array_equal(dd["val_codes"].cpu().numpy(), vc)
    out, lse = run_gpu(d2, dd=dd)
    ref_out, ref_lse = run_oracle(d2)
    assert_close(out, lse, ref_out, ref_lse)


def test_full_size_batch16():
    """The ragged 16-sequence LLaMA-3.1-8B layer (8 KV heads, R = 2): every sequence
    appends at its own length."""
    w = workloads.WORKLOADS["llama8b_batch16_ragged_R2_zipf"]
    d = workloads.generate(w, t_cap=64)
    d["seq_lens"] = np.random.default_rng(75).integers(0, 64, size=w.batch).astype(np.int32)
    rng = np.random.default_rng(75)
    keys, vals = _new_vectors(rng, d, True)
    gk, gv, ok, ov = _run(d, keys, vals, d["seq_lens"])
    assert np.array_equal(gk, ok) and np.array_equal(gv, ov)


# ---------------------------------------------------------------------------
# the paper's layout: 2 groups of 64 scalars, 64 codewords, planar codes [B, Hkv, 2, R, T]
# ---------------------------------------------------------------------------
def _wide_case(R, T, lens, seed):
    return workloads.small(batch=len(lens), n_q_heads=8, n_kv_heads=2, t_cap=T, R=R,
                           seq_lens=np.asarray(lens, np.int32), seed=seed,
                           cb_std=math.sqrt(1.0 / R), group_dim=64)


@pytest.mark.parametrize("R", [1, 11, 21])
def test_wide_codes_bit_exact(R):
    d = _wide_case(R, 48, [48, 48, 48], seed=80 + R)
    rng = np.random.default_rng(800 + R)
    keys = rng.standard_normal((3, 2, 128), dtype=np.float32)
    vals = rng.standard_normal((3, 2, 128), dtype=np.float32)
    positions = np.array([0, 47, -3], np.int32)
    kc = np.full(d["key_codes"].shape, FILL, np.uint8)
    vc = np.full(d["val_codes"].shape, FILL, np.uint8)
    dk, dv = torch.from_numpy(kc.copy()).cuda(), torch.from_numpy(vc.copy()).cuda()
    shape = cvq.make_shape(3, 8, 2, R, 48, d["rope_base"], 128, 64)
    cvq.encode_append(shape, torch.from_numpy(keys).cuda(), torch.from_numpy(vals).cuda(),
                      torch.from_numpy(d["key_cb"]).cuda(), torch.from_numpy(d["val_cb"]).cuda(),
                      torch.from_numpy(positions).cuda(), dk, dv)
    torch.cuda.synchronize()
    E.encode_append(keys, vals, d["key_cb"], d["val_cb"], positions, kc, vc, codes_layout="planar")
    gk, gv = dk.cpu().numpy(), dv.cpu().numpy()
    assert np.array_equal(gk, kc) and np.array_equal(gv, vc)
    assert np.all(gk[2] == FILL) and int(gk[0, :, :, :, 0].max()) < 64


def test_wide_append_then_attend_matches_oracle():
    d = _wide_case(11, 512, [300, 511], seed=85)
    rng = np.random.default_rng(85)
    keys = rng.standard_normal((2, 2, 128), dtype=np.float32)
    vals = rng.standard_normal((2, 2, 128), dtype=np.float32)
    dd = to_device(d)
    shape = cvq.shape_of(dd["q"], dd["key_codes"], d["rope_base"], 64)
    cvq.encode_append(shape, torch.from_numpy(keys).cuda(), torch.from_numpy(vals).cuda(),
                      dd["key_cb"], dd["val_cb"], dd["seq_lens"].clone(), dd["key_codes"],
                      dd["val_codes"])
    dd["seq_lens"] += 1
    kc, vc = d["key_codes"].copy(), d["val_codes"].copy()
    E.encode_append(keys, vals, d["key_cb"], d["val_cb"], d["seq_lens"], kc, vc,
                    codes_layout="planar")
    d2 = dict(d, key_codes=kc, val_codes=vc, seq_lens=d["seq_lens"] + 1)
    assert np.array_equal(dd["key_codes"].cpu().numpy(), kc)
    assert np.array_equal(dd["val_codes"].cpu().numpy(), vc)
    out, lse = run_gpu(d2, dd=dd)
    ref_out, ref_lse = run_oracle(d2)
    assert_close(out, lse, ref_out, ref_lse)
