"""GPU checks of cvq_attend: the GQA decode with the split merge fused into the last CTA
of every work unit (one launch per decode step).

- against the float64 oracle, to the usual bar (max |out - oracle| <= 2e-3, lse relative
  error <= 1e-4), for every kernel that carries the fused merge: the clustered 4-head
  kernel (R = 1, 2), the plain kernel (1, 2 and 8 query heads per KV head) and the
  64-scalar-group kernel (R = 11, 21), with ragged lengths and empty splits;
- bit for bit against cvq_combine run on the partial states the fused call left in its
  workspace (the merge arithmetic is the same, in the same order);
- the arrival counters are zero again after every call, so a workspace is reusable.
"""
import ctypes
import math

import numpy as np
import pytest

import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import compressed_attention_cvq_b200 as cvq
    from compressed_attention_cvq_b200 import _binding as _b
    from gpu_util import assert_close, run_oracle, to_device

CASES = [
    # (group, R, group_dim, T, lens, splits)
    (4, 1, 8, 1500, [1500, 700, 0], 5),
    (4, 2, 8, 2048, [2048, 64], 6),
    (1, 1, 8, 900, [900, 17, 333], 4),
    (2, 2, 8, 640, [640, 100, 1], 3),
    (8, 1, 8, 512, [512, 500, 0], 2),
    (4, 11, 64, 1024, [1024, 300, 0], 4),
    (4, 21, 64, 768, [768, 129, 5], 3),
    (4, 1, 8, 4480, [4480, 2100, 64], 70),   # more than 32 splits: the merge reloads m, l
    (1, 2, 8, 2112, [2112, 2049, 0], 33),
]


def _case(group, R, gd, T, lens, seed):
    return workloads.small(batch=len(lens), n_q_heads=2 * group, n_kv_heads=2, t_cap=T, R=R,
                           seq_lens=np.asarray(lens, np.int32), seed=seed,
                           cb_std=math.sqrt(1.0 / R), group_dim=gd)


@pytest.mark.parametrize("group,R,gd,T,lens,splits", CASES)
def test_fused_matches_oracle_and_combine(group, R, gd, T, lens, splits):
    d = _case(group, R, gd, T, lens, seed=90 + group + R)
    dd = to_device(d)
    shape = cvq.shape_of(dd["q"], dd["key_codes"], d["rope_base"], gd)
    ws = cvq.workspace_alloc(shape, splits, "cuda")
    for _ in range(3):                       # the counters reset: the workspace is reusable
        out, lse = cvq.attend_fused(shape, dd["q"], dd["key_cb"], dd["key_codes"], dd["val_codes"],
                                    dd["seq_lens"], dd["val_cb"], splits, workspace=ws)
    torch.cuda.synchronize()
    B, Hq = shape.batch, shape.n_q_heads
    rows = B * Hq * splits
    counters = ws[rows * 130 * 4:].view(torch.int32)
    assert int(counters.abs().sum()) == 0
    # the merge of cvq_combine on the partials this call left in the workspace: same bits
    wsf = ws[: rows * 130 * 4].view(torch.float32)
    po = wsf[: rows * 128]
    pm = wsf[rows * 128: rows * 129]
    pl = wsf[rows * 129:]
    out2, lse2 = cvq.combine(shape, splits, po, pm, pl)
    torch.cuda.synchronize()
    assert torch.equal(out, out2) and torch.equal(lse, lse2)
    ref_out, ref_lse = run_oracle(d)
    assert_close(out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
                 ref_out, ref_lse)


def test_fused_full_size_128k():
    """The 128K-token LLaMA-3.1-8B layer (R = 1) in the benchmark's configuration."""
    w = workloads.WORKLOADS["llama8b_layer_T131072_R1"]
    d = workloads.generate(w)
    dd = to_device(d)
    out, lse = cvq.attend(dd["q"], dd["key_cb"], dd["val_cb"], dd["key_codes"], dd["val_codes"],
                          dd["seq_lens"], d["rope_base"], form="gqa")
    torch.cuda.synchronize()
    heads = [(0, 3), (0, 17), (0, 30)]
    ref_out, ref_lse = run_oracle(d, heads=heads)
    assert_close(out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
                 ref_out, ref_lse, heads=heads)


@pytest.mark.gpu
def test_128k_layer_with_one_and_two_splits():
    """The 128K-token layer decoded with 1 and 2 splits: each CTA pair walks 64K-128K
    positions, 256 to 512 tiles, so the RoPE phase must stay exact over a long split (it is
    re-seeded from the exact fixed-point turn at every tile and advanced within it)."""
    w = workloads.WORKLOADS["llama8b_layer_T131072_R1"]
    d = workloads.generate(w)
    dd = to_device(d)
    heads = [(0, 1), (0, 14), (0, 31)]
    ref_out, ref_lse = run_oracle(d, heads=heads)
    for n_splits in (1, 2):
        out, lse = cvq.attend(dd["q"], dd["key_cb"], dd["val_cb"], dd["key_codes"],
                              dd["val_codes"], dd["seq_lens"], d["rope_base"], n_splits=n_splits,
                              form="gqa")
        torch.cuda.synchronize()
        assert_close(out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
                     ref_out, ref_lse, heads=heads)


def test_rope_base_change_between_calls():
    """The library keeps the phase increments of the last RoPE base a thread asked for: calls
    that alternate between two bases (500000 and 10000) each match the oracle run with their
    own base."""
    lens = [1200, 777]
    cases = {base: _case_base(base, lens) for base in (500000.0, 10000.0)}
    for base in (500000.0, 10000.0, 500000.0, 10000.0):
        d, dd = cases[base]
        out, lse = cvq.attend(dd["q"], dd["key_cb"], dd["val_cb"], dd["key_codes"], dd["val_codes"],
                              dd["seq_lens"], base, n_splits=3)
        torch.cuda.synchronize()
        ref_out, ref_lse = run_oracle(d)
        assert_close(out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
                     ref_out, ref_lse)


def _case_base(base, lens):
    d = workloads.small(batch=len(lens), n_q_heads=8, n_kv_heads=2, t_cap=1280, R=1,
                        seq_lens=np.asarray(lens, np.int32), seed=97, rope_base=base)
    return d, to_device(d)
