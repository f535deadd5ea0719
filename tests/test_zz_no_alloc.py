"""cvq_attend_static: the decode step for callers that cannot allocate device memory
while decoding (a server whose pool already holds all free HBM for the KV cache, a
plugin without an allocator, a loop that cannot take cudaMalloc's implicit sync).

The entry point keeps its split partial states in a fixed device array inside the
library.  Called directly through the C ABI, its out and lse must match the
caller-allocated path (cvq_decode_attn_gqa + cvq_combine) on two calls in a row with
different inputs, and a call whose partials do not fit must be refused before any
launch.  This file is collected last so that a failure here comes after every other
test has run.
"""
import ctypes

import numpy as np
import pytest

import workloads
from compressed_attention_cvq_b200 import _binding as b

OUT_TOL = 2e-3
LSE_RTOL = 1e-4


def _shape(B, Hq, Hkv, R, T):
    return b.make_shape(B, Hq, Hkv, R, T)


def test_static_limit_refused_before_launch():
    # 64 x 32 x 64 rows x 130 floats x 4 B = 68 MB > 4 MiB; the pointers are never used
    s = _shape(64, 32, 8, 1, 8192)
    fake = 0x10000
    st = b.lib.cvq_attend_static(ctypes.byref(s), fake, 0, fake, 0, fake, fake, fake, fake, 0,
                                 64, fake, fake, None)
    assert st == 7 and b.status_str(st).startswith("CVQ_ERR_STATIC_LIMIT")


@pytest.mark.gpu
def test_static_matches_allocated_path_twice():
    import torch

    import compressed_attention_cvq_b200 as cvq
    from gpu_util import to_device

    cases = [
        workloads.small(batch=2, n_q_heads=8, n_kv_heads=2, t_cap=1500, R=2, q_dtype="bf16",
                        seq_lens=np.array([1500, 700], np.int32), seed=101, cb_std=0.7071),
        workloads.small(batch=1, n_q_heads=32, n_kv_heads=8, t_cap=4096, R=1, seed=202),
    ]
    for d in cases:
        dd = to_device(d)
        shape = cvq.shape_of(dd["q"], dd["key_codes"], d["rope_base"])
        S = cvq.suggest_splits(shape)
        ref_out, ref_lse = cvq.combine(shape, S, *cvq.decode_attn_gqa(
            shape, dd["q"], dd["key_cb"], dd["key_codes"], dd["val_codes"], dd["seq_lens"],
            dd["val_cb"], S))
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        q_dtype = 1 if dd["q"].dtype == torch.bfloat16 else 0
        st = b.lib.cvq_attend_static(
            ctypes.byref(shape), dd["q"].data_ptr(), q_dtype, dd["key_cb"].data_ptr(),
            dd["key_cb"].numel() // dd["key_cb"].shape[0], dd["key_codes"].data_ptr(),
            dd["val_codes"].data_ptr(), dd["seq_lens"].data_ptr(), dd["val_cb"].data_ptr(),
            dd["val_cb"].numel() // dd["val_cb"].shape[0], S, out.data_ptr(), lse.data_ptr(),
            torch.cuda.current_stream().cuda_stream)
        assert st == 0, b.status_str(st)
        torch.cuda.synchronize()
        o, l = out.cpu().numpy(), lse.cpu().numpy()
        ro, rl = ref_out.cpu().numpy(), ref_lse.cpu().numpy()
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(l))
        assert np.max(np.abs(o - ro)) <= OUT_TOL
        assert np.max(np.abs(l - rl) / np.maximum(np.abs(rl), 1.0)) <= LSE_RTOL
