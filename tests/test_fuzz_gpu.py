"""Randomized GPU parity: many small shapes drawn from a fixed seed, across every decode
path the library has (GQA one-launch, GQA + combine, table form), both group sizes, both
query dtypes, ragged and empty sequences, and split counts from 1 up to more splits than
the sequences have 64-token blocks.  Each case is compared with the float64 oracle to the
usual bar (max |out - oracle| <= 2e-3, lse relative error <= 1e-4).
"""
import math

import numpy as np
import pytest

import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from gpu_util import assert_close, run_gpu, run_oracle


def _draw(i):
    rng = np.random.default_rng(1000 + i)
    wide = rng.random() < 0.3
    if wide:
        group, R = 4, int(rng.integers(1, 23))
        T = 16 * int(rng.integers(1, 48))
    else:
        group = int(rng.choice([1, 2, 4, 8]))
        R = int(rng.integers(1, 3)) if group * 2 <= 8 else 1
        T = int(rng.integers(1, 700))
    B = int(rng.integers(1, 4))
    Hkv = int(rng.integers(1, 4))
    lens = rng.integers(0, T + 1, size=B).astype(np.int32)
    if rng.random() < 0.5:
        lens[int(rng.integers(0, B))] = T                       # one full-length sequence
    splits = int(rng.integers(1, 9))
    if rng.random() < 0.2:
        splits = int(rng.integers(9, 40))                       # many (mostly empty) splits
    forms = ["gqa", "gqa_split"] + ([] if wide else ["table"])
    form = forms[int(rng.integers(0, len(forms)))]
    q_dtype = "bf16" if rng.random() < 0.4 else "f32"
    return dict(group=group, R=R, T=T, B=B, Hkv=Hkv, lens=lens, splits=splits, form=form,
                q_dtype=q_dtype, gd=64 if wide else 8, seed=2000 + i)


@pytest.mark.parametrize("i", range(100))
def test_fuzz(i):
    c = _draw(i)
    d = workloads.small(batch=c["B"], n_q_heads=c["group"] * c["Hkv"], n_kv_heads=c["Hkv"],
                        t_cap=c["T"], R=c["R"], q_dtype=c["q_dtype"], seq_lens=c["lens"],
                        seed=c["seed"], cb_std=math.sqrt(1.0 / c["R"]), group_dim=c["gd"])
    out, lse = run_gpu(d, form=c["form"], n_splits=c["splits"])
    ref_out, ref_lse = run_oracle(d)
    assert_close(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("i", range(30))
def test_fuzz_encode_append(i):
    """The write side on random shapes: codes bit-exact with the oracle's, nothing else
    written."""
    import compressed_attention_cvq_b200 as cvq
    from oracle import encode as E

    rng = np.random.default_rng(3000 + i)
    wide = rng.random() < 0.4
    R = int(rng.integers(1, 23)) if wide else int(rng.integers(1, 3))
    B, Hkv = int(rng.integers(1, 5)), int(rng.integers(1, 4))
    T = 16 * int(rng.integers(1, 6)) if wide else int(rng.integers(1, 80))
    d = workloads.small(batch=B, n_q_heads=4 * Hkv, n_kv_heads=Hkv, t_cap=T, R=R, seed=4000 + i,
                        cb_std=math.sqrt(1.0 / R), group_dim=64 if wide else 8)
    keys = rng.standard_normal((B, Hkv, 128)).astype(np.float32)
    vals = rng.standard_normal((B, Hkv, 128)).astype(np.float32)
    pos = rng.integers(-2, T + 2, size=B).astype(np.int32)
    kc = np.full(d["key_codes"].shape, 0x5A, np.uint8)
    vc = np.full(d["val_codes"].shape, 0x5A, np.uint8)
    dk, dv = torch.from_numpy(kc.copy()).cuda(), torch.from_numpy(vc.copy()).cuda()
    shape = cvq.make_shape(B, 4 * Hkv, Hkv, R, T, d["rope_base"], 128, 64 if wide else 8)
    cvq.encode_append(shape, torch.from_numpy(keys).cuda(), torch.from_numpy(vals).cuda(),
                      torch.from_numpy(d["key_cb"]).cuda(), torch.from_numpy(d["val_cb"]).cuda(),
                      torch.from_numpy(pos).cuda(), dk, dv)
    torch.cuda.synchronize()
    E.encode_append(keys, vals, d["key_cb"], d["val_cb"], pos, kc, vc,
                    codes_layout="planar" if wide else "token")
    assert np.array_equal(dk.cpu().numpy(), kc) and np.array_equal(dv.cpu().numpy(), vc)


@pytest.mark.parametrize("i", range(12))
def test_fuzz_larger(i):
    """Fewer, larger random cases: several tiles per split, up to 8 KV heads, up to 200
    splits (the fused merge walks many partial states)."""
    rng = np.random.default_rng(5000 + i)
    wide = rng.random() < 0.3
    group = 4 if wide else int(rng.choice([1, 2, 4, 8]))
    R = int(rng.integers(1, 23)) if wide else (1 if group == 8 else int(rng.integers(1, 3)))
    T = 16 * int(rng.integers(64, 320)) if wide else int(rng.integers(1000, 5000))
    B, Hkv = int(rng.integers(1, 4)), int(rng.integers(1, 9))
    lens = rng.integers(0, T + 1, size=B).astype(np.int32)
    lens[0] = T
    splits = int(rng.integers(1, 201))
    d = workloads.small(batch=B, n_q_heads=group * Hkv, n_kv_heads=Hkv, t_cap=T, R=R,
                        q_dtype="bf16" if rng.random() < 0.5 else "f32", seq_lens=lens,
                        seed=6000 + i, cb_std=math.sqrt(1.0 / R), group_dim=64 if wide else 8)
    out, lse = run_gpu(d, form="gqa", n_splits=splits)
    heads = [(b, h) for b in range(B) for h in rng.choice(group * Hkv, size=min(6, group * Hkv),
                                                           replace=False)]
    ref_out, ref_lse = run_oracle(d, heads=heads)
    assert_close(out, lse, ref_out, ref_lse, heads=heads)
