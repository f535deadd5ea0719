"""GPU parity of the naive comparison path (decode the cache to fp16, then attend).

The dequantized keys and values must equal the oracle's reconstruction (keys rotated by
RoPE) to fp16 rounding; the attention over them must match the float64 oracle within the
path's tolerance (max |out - oracle| <= 2e-3, lse rel <= 1e-4): fp16 keys and values add
~2.4e-4 relative rounding per element on top of the fp32 arithmetic.
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


@pytest.mark.parametrize("R", [1, 2])
def test_dequant_matches_oracle_reconstruction(R):
    lens = np.array([300, 77], np.int32)
    d = workloads.small(batch=2, n_q_heads=8, n_kv_heads=2, t_cap=300, R=R, seq_lens=lens, seed=40 + R,
                        cb_std=math.sqrt(1.0 / R))
    dd = to_device(d)
    shape = cvq.shape_of(dd["q"], dd["key_codes"])
    k, v = cvq.naive_dequant(shape, dd["key_cb"], dd["val_cb"], dd["key_codes"], dd["val_codes"],
                             dd["seq_lens"])
    k, v = k.float().cpu().numpy(), v.float().cpu().numpy()
    theta = O.rope_theta(d["rope_base"])
    for b in range(2):
        for h in range(2):
            L = int(lens[b])
            rk = O.apply_rope(O.decode_keys(d["key_cb"][h], d["key_codes"][b, h, :L]), np.arange(L), theta)
            vv = O.decode_values(d["val_cb"][h], d["val_codes"][b, h, :L])
            np.testing.assert_allclose(k[b, h, :L], rk, rtol=2 ** -10, atol=1e-5)
            np.testing.assert_allclose(v[b, h, :L], vv, rtol=2 ** -10, atol=1e-6)
            assert np.all(k[b, h, L:] == 0) and np.all(v[b, h, L:] == 0)   # untouched


@pytest.mark.parametrize("group,R,T", [(1, 1, 1000), (4, 1, 777), (4, 2, 1500), (2, 2, 65)])
def test_naive_attention_matches_oracle(group, R, T):
    d = workloads.small(batch=2, n_q_heads=2 * group, n_kv_heads=2, t_cap=T, R=R,
                        seq_lens=np.array([T, T // 3], np.int32), seed=50 + R + group,
                        cb_std=math.sqrt(1.0 / R))
    out, lse = run_gpu(d, form="naive", n_splits=3)
    ref_out, ref_lse = run_oracle(d)
    assert_close(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("name,k", [("llama8b_layer_T131072_R1", 4), ("llama8b_layer_T32768_R2", 8)])
def test_naive_full_size(name, k):
    w = workloads.WORKLOADS[name]
    d = workloads.generate(w)
    out, lse = run_gpu(d, form="naive", n_splits=74)
    rng = np.random.default_rng(1)
    heads = [(0, int(h)) for h in rng.choice(w.n_q_heads, size=k, replace=False)]
    ref_out, ref_lse = run_oracle(d, heads=heads)
    assert_close(out, lse, ref_out, ref_lse, heads=heads)
