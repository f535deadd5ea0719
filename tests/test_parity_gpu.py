"""GPU parity: the library's kernels against the float64 oracle on identical seeded
inputs.  Tolerances: max |out - oracle| <= 2e-3 and |lse - oracle| / max(|oracle|, 1)
<= 1e-4 (fp32 kernels against a float64 definition); the P table to fp32 rounding.

Small cases span several 256-token tiles with ragged tails, empty splits, empty
sequences, every GQA group size, both residual depths, shared codebooks, bf16 queries
and Zipf-skewed codes.  The five full-size workloads run in the benchmark's launch
configuration and are compared on sampled heads.
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


FORMS = ["gqa", "table"]


def _small(**kw):
    return workloads.small(**kw)


@pytest.mark.parametrize("q_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("R", [1, 2])
def test_qtable_matches_oracle(q_dtype, R):
    d = _small(batch=2, n_q_heads=8, n_kv_heads=2, t_cap=8, R=R, q_dtype=q_dtype, seed=3)
    dd = to_device(d)
    shape = cvq.shape_of(dd["q"], dd["key_codes"])
    P = cvq.qtable(shape, dd["q"], dd["key_cb"]).cpu().numpy().astype(np.float64)
    ref = O.qtable(d["q"], d["key_cb"], 2)
    np.testing.assert_allclose(P, ref, rtol=0, atol=2e-6 * max(1.0, np.abs(ref).max()))


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 255, 256, 257, 1000, 3001])
def test_lengths_and_tails(form, T):
    d = _small(batch=1, n_q_heads=4, n_kv_heads=1, t_cap=T, R=1, seed=T)
    out, lse = run_gpu(d, form=form, n_splits=3)
    ref_out, ref_lse = run_oracle(d)
    assert_close(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("group,R", [(1, 1), (1, 2), (2, 1), (2, 2), (4, 1), (4, 2), (8, 1)])
def test_gqa_groups_and_rounds(form, group, R):
    d = _small(batch=2, n_q_heads=2 * group, n_kv_heads=2, t_cap=777, R=R, seed=10 * group + R,
               cb_std=math.sqrt(1.0 / R))
    out, lse = run_gpu(d, form=form, n_splits=2)
    ref_out, ref_lse = run_oracle(d)
    assert_close(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("n_splits", [1, 2, 5, 16, 40])
def test_split_counts_including_empty_splits(form, n_splits):
    d = _small(batch=1, n_q_heads=4, n_kv_heads=1, t_cap=1500, R=2, seed=n_splits,
               cb_std=math.sqrt(0.5))
    out, lse = run_gpu(d, form=form, n_splits=n_splits)
    ref_out, ref_lse = run_oracle(d)
    assert_close(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("form", FORMS)
def test_ragged_batch_with_empty_and_short_sequences(form):
    lens = np.array([0, 1, 64, 65, 2000, 1999, 3, 0], dtype=np.int32)
    d = _small(batch=8, n_q_heads=8, n_kv_heads=2, t_cap=2000, R=2, seq_lens=lens, seed=77,
               cb_std=math.sqrt(0.5), codes="zipf1.1")
    out, lse = run_gpu(d, form=form, n_splits=4)
    ref_out, ref_lse = run_oracle(d)
    assert_close(out, lse, ref_out, ref_lse)
    assert np.all(np.isneginf(lse[0])) and np.all(out[0] == 0)


@pytest.mark.parametrize("form", FORMS)
def test_bf16_queries_and_shared_codebooks(form):
    d = _small(batch=2, n_q_heads=8, n_kv_heads=2, t_cap=600, R=2, q_dtype="bf16", seed=5,
               cb_std=math.sqrt(0.5))
    # one codebook shared by both KV heads: pass it without the head dim (stride 0)
    d["key_cb"] = np.repeat(d["key_cb"][:1], 2, axis=0)
    d["val_cb"] = np.repeat(d["val_cb"][:1], 2, axis=0)
    dd = to_device(d)
    dd["key_cb"] = dd["key_cb"][0].contiguous()
    dd["val_cb"] = dd["val_cb"][0].contiguous()
    out, lse = run_gpu(d, form=form, n_splits=2, dd=dd)
    ref_out, ref_lse = run_oracle(d)
    assert_close(out, lse, ref_out, ref_lse)


def test_seq_lens_clamped_to_capacity():
    d = _small(batch=2, n_q_heads=4, n_kv_heads=1, t_cap=300, R=1, seed=8,
               seq_lens=np.array([300, 300], np.int32))
    dd = to_device(d)
    dd["seq_lens"] = torch.tensor([5000, -3], dtype=torch.int32, device="cuda")
    out, lse = run_gpu(d, n_splits=2, dd=dd)
    d["seq_lens"] = np.array([300, 0], np.int32)
    ref_out, ref_lse = run_oracle(d)
    assert_close(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("form", FORMS)
def test_partials_follow_documented_split_rule(form):
    """Each split's (m, l, o) is the oracle's partial state over tokens
    [s*C, min((s+1)*C, L)), C = cvq_split_tokens, up to the choice of reference m."""
    d = _small(batch=1, n_q_heads=4, n_kv_heads=1, t_cap=1000, R=1, seed=21)
    dd = to_device(d)
    shape = cvq.shape_of(dd["q"], dd["key_codes"])
    S = 3
    if form == "gqa":
        po, pm, pl = cvq.decode_attn_gqa(shape, dd["q"], dd["key_cb"], dd["key_codes"],
                                         dd["val_codes"], dd["seq_lens"], dd["val_cb"], S)
    else:
        P = cvq.qtable(shape, dd["q"], dd["key_cb"])
        po, pm, pl = cvq.decode_attn(shape, P, dd["key_codes"], dd["val_codes"], dd["seq_lens"],
                                     dd["val_cb"], S)
    po, pm, pl = (x.cpu().numpy().astype(np.float64) for x in (po, pm, pl))
    C = cvq.split_tokens(shape, S)
    bounds = [(s * C, min((s + 1) * C, 1000)) for s in range(S)]
    for hq in range(4):
        s = O.scores(d["q"][0, hq], d["key_cb"][0], d["key_codes"][0, 0], 1000, d["rope_base"])
        v = O.decode_values(d["val_cb"][0], d["val_codes"][0, 0])
        m, l, o = O.split_partials(s, v, bounds)
        for si, (t0, t1) in enumerate(bounds):
            if t1 <= t0:
                assert np.isneginf(pm[0, hq, si]) and pl[0, hq, si] == 0
                continue
            # m is a reference point within [max - 8 ln 2, max]; the split's log-sum-exp
            # m + ln l and its normalized output o / l do not depend on that choice
            assert m[si] - 8 * math.log(2) - 1e-4 <= pm[0, hq, si] <= m[si] + 1e-4
            lse_gpu = pm[0, hq, si] + math.log(pl[0, hq, si])
            lse_ref = m[si] + math.log(l[si])
            assert abs(lse_gpu - lse_ref) / max(1.0, abs(lse_ref)) < 1e-4
            np.testing.assert_allclose(po[0, hq, si] / pl[0, hq, si], o[si] / l[si], atol=2e-3)


def test_combine_matches_oracle_merge():
    rng = np.random.default_rng(4)
    B, Hq, S = 2, 4, 7
    m = rng.standard_normal((B, Hq, S)) * 3
    m[0, 0, 2] = -np.inf
    m[1, 2, :] = -np.inf  # a head whose every split is empty
    l = rng.random((B, Hq, S)) * 50 + 0.5
    l[np.isneginf(m)] = 0
    o = rng.standard_normal((B, Hq, S, 128)) * 10
    o[np.isneginf(m)] = 0
    shape = cvq.make_shape(B, Hq, 1, 1, 64)
    t = lambda x: torch.from_numpy(x.astype(np.float32)).cuda()
    out, lse = cvq.combine(shape, S, t(o), t(m), t(l))
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for b in range(B):
        for h in range(Hq):
            ro, rl = O.combine(m[b, h].astype(np.float32), l[b, h].astype(np.float32),
                               o[b, h].astype(np.float32))
            if np.isneginf(rl):
                assert np.isneginf(lse[b, h]) and np.all(out[b, h] == 0)
            else:
                np.testing.assert_allclose(out[b, h], ro, rtol=1e-5, atol=1e-5)
                assert abs(lse[b, h] - rl) < 1e-5 * max(1, abs(rl))


# ---------------------------------------------------------------------------
# the five full-size workloads, in the benchmark's launch configuration
# ---------------------------------------------------------------------------
def _sample_heads(B, Hq, k, seed):
    rng = np.random.default_rng(seed)
    allh = [(b, h) for b in range(B) for h in range(Hq)]
    if len(allh) <= k:
        return allh
    idx = rng.choice(len(allh), size=k, replace=False)
    return [allh[i] for i in sorted(idx)]


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("name,layers,k", [
    ("single_head_T4096_R1", [0], 1),
    ("llama8b_layer_T32768_R2", [0], 32),
    ("llama8b_layer_T131072_R1", [0], 6),
    ("llama8b_batch16_ragged_R2_zipf", [0], 24),
    ("llama8b_32layers_B4_T65536_R2", [0, 31], 4),
])
def test_full_size_workloads(form, name, layers, k):
    w = workloads.WORKLOADS[name]
    for layer in layers:
        d = workloads.generate(w, layer=layer)
        out, lse = run_gpu(d, form=form)          # default split count, as the bench uses
        heads = _sample_heads(w.batch, w.n_q_heads, k, seed=layer)
        ref_out, ref_lse = run_oracle(d, heads=heads)
        assert_close(out, lse, ref_out, ref_lse, heads=heads)
        # every head: finite, weights form a distribution (lse >= max possible single score)
        assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
