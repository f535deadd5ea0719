"""GPU checks of the codebook staging by the TMA engine.

The 4-query-head kernel copies its half of each codebook through a 5-d tiled tensor map
(groups x codeword halves x codes x heads) straight into its bank-conflict-free chunk
layout; the 64-scalar-group kernel copies its rounds with one bulk copy.  Both take the
codebook's head stride from the caller, so these cases give the codebooks padded head
strides (heads further apart than one codebook, a different pad for keys and values) and
a stride of 0 (one codebook for all heads), call the C ABI directly, and compare with the
float64 oracle to the usual bar (max |out - oracle| <= 2e-3, lse relative error <= 1e-4).
The library's device fault word (set by a bounded copy wait that gives up) must stay 0.
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


def _padded(cb, pad):
    """A [H, ...] codebook copied into a buffer whose heads are numel/H + pad floats apart:
    (base tensor, head stride in floats)."""
    H = cb.shape[0]
    per = cb[0].numel()
    buf = torch.full((H, per + pad), float("nan"), dtype=torch.float32, device="cuda")
    buf[:, :per] = cb.reshape(H, per)
    return buf, per + pad


def _attend_raw(d, dd, key_base, key_stride, val_base, val_stride, n_splits, group_dim):
    shape = cvq.shape_of(dd["q"], dd["key_codes"], d["rope_base"], group_dim)
    ws = cvq.workspace_alloc(shape, n_splits, dd["q"].device)
    B, Hq = dd["q"].shape[:2]
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    q_dtype = 1 if dd["q"].dtype == torch.bfloat16 else 0
    st = _b.lib.cvq_attend(ctypes.byref(shape), dd["q"].data_ptr(), q_dtype, key_base.data_ptr(),
                           key_stride, dd["key_codes"].data_ptr(), dd["val_codes"].data_ptr(),
                           dd["seq_lens"].data_ptr(), val_base.data_ptr(), val_stride, n_splits,
                           ws.data_ptr(), out.data_ptr(), lse.data_ptr(), None)
    assert st == 0, _b.status_str(st)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("R,kpad,vpad", [(1, 4, 12), (2, 64, 4), (1, 0, 0)])
def test_gqa4_padded_head_strides(R, kpad, vpad):
    d = workloads.small(batch=2, n_q_heads=12, n_kv_heads=3, t_cap=1300, R=R, seed=90 + R + kpad,
                        seq_lens=np.array([1300, 611], np.int32), cb_std=math.sqrt(1.0 / R),
                        q_dtype="bf16" if R == 2 else "f32")
    dd = to_device(d)
    kb, ks = _padded(dd["key_cb"], kpad)
    vb, vs = _padded(dd["val_cb"], vpad)
    out, lse = _attend_raw(d, dd, kb, ks, vb, vs, 5, 8)
    ref_out, ref_lse = run_oracle(d)
    assert_close(out, lse, ref_out, ref_lse)
    assert cvq.fault_status(clear=True) == 0


@pytest.mark.parametrize("R", [1, 2])
def test_gqa4_one_codebook_for_all_heads(R):
    d = workloads.small(batch=1, n_q_heads=16, n_kv_heads=4, t_cap=900, R=R, seed=97 + R,
                        cb_std=math.sqrt(1.0 / R))
    d["key_cb"] = np.repeat(d["key_cb"][:1], 4, axis=0)
    d["val_cb"] = np.repeat(d["val_cb"][:1], 4, axis=0)
    dd = to_device(d)
    out, lse = _attend_raw(d, dd, dd["key_cb"][0].contiguous(), 0, dd["val_cb"][0].contiguous(), 0,
                           3, 8)
    ref_out, ref_lse = run_oracle(d)
    assert_close(out, lse, ref_out, ref_lse)
    assert cvq.fault_status(clear=True) == 0


@pytest.mark.parametrize("R,kpad,vpad", [(11, 8, 4), (21, 4, 32)])
def test_wide_padded_head_strides(R, kpad, vpad):
    d = workloads.small(batch=2, n_q_heads=8, n_kv_heads=2, t_cap=768, R=R, seed=120 + R,
                        seq_lens=np.array([768, 300], np.int32), cb_std=math.sqrt(1.0 / R),
                        group_dim=64)
    dd = to_device(d)
    kb, ks = _padded(dd["key_cb"], kpad)
    vb, vs = _padded(dd["val_cb"], vpad)
    out, lse = _attend_raw(d, dd, kb, ks, vb, vs, 3, 64)
    ref_out, ref_lse = run_oracle(d)
    assert_close(out, lse, ref_out, ref_lse)
    assert cvq.fault_status(clear=True) == 0


def test_fault_word_starts_and_stays_clear():
    d = workloads.small(batch=1, n_q_heads=4, n_kv_heads=1, t_cap=512, R=1, seed=130)
    dd = to_device(d)
    per = dd["key_cb"][0].numel()
    out, lse = _attend_raw(d, dd, dd["key_cb"], per, dd["val_cb"], per, 2, 8)
    ref_out, ref_lse = run_oracle(d)
    assert_close(out, lse, ref_out, ref_lse)
    assert cvq.fault_status() == 0
    assert cvq.fault_status(clear=True) == 0
