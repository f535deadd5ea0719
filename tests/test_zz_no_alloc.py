"""cvq_attend_static: the decode step for callers that cannot allocate device memory while
decoding -- a server whose memory pool already holds all free HBM for the KV cache, a
plugin whose host gives it no allocator, a decode loop that cannot take cudaMalloc's
implicit synchronization.

The entry point keeps its arrival counters and split partial states in one fixed device
array inside the library (counters in a fixed region at its start, partial states after
it) and clears the counters it uses at every call.  Called directly through the C ABI,
calls of different shapes in any order must each match the float64 oracle and
cvq_attend (the caller-allocated path, on a freshly zeroed workspace) within the parity
tolerance -- not bit for bit: the value bins are summed with float atomics whose order
varies from run to run; a call that does not fit must be refused before any launch.  This file is collected last so
that a failure here comes after every other test has run; its GPU test also passes when
run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest

import workloads
from compressed_attention_cvq_b200 import _binding as b

OUT_TOL = 2e-3
LSE_RTOL = 1e-4
STATIC_BYTES = 4 * 1024 * 1024
COUNTER_BYTES = 32 * 1024


def _shape(B, Hq, Hkv, R, T, group_dim=8):
    s = b.make_shape(B, Hq, Hkv, R, T)
    s.group_dim = group_dim
    return s


def _call_static(s, fake=0x10000, n_splits=1, q_dtype=0):
    # fake pointers: every call here must be refused on the host before any launch
    return b.lib.cvq_attend_static(ctypes.byref(s), fake, q_dtype, fake, 0, fake, fake, fake,
                                   fake, 0, n_splits, fake, fake, None)


def test_static_limit_refused_before_launch():
    # 64 x 32 x 64 rows x 130 floats x 4 B = 68 MB > 4 MiB; the pointers are never used
    st = _call_static(_shape(64, 32, 8, 1, 8192), n_splits=64)
    assert st == 7 and b.status_str(st).startswith("CVQ_ERR_STATIC_LIMIT")


def test_static_limit_counts_the_counter_region():
    # the partial states get the array minus its 32 KiB counter region: a row (sequence,
    # query head, split) takes 130 floats = 520 B, so 8002 rows fit and 8003 do not
    room = STATIC_BYTES - COUNTER_BYTES
    fit_rows = room // 520
    assert fit_rows == 8002 and fit_rows * 520 <= room < (fit_rows + 1) * 520
    # rows = batch x query heads x splits; here batch = rows, one head, one split
    s_fit = _shape(fit_rows, 1, 1, 1, 64)
    s_over = _shape(fit_rows + 1, 1, 1, 1, 64)
    assert b.lib.cvq_partials_bytes(ctypes.byref(s_fit), 1) == fit_rows * 520
    assert _call_static(s_over) == 7
    # the call that fits passes the size check and is then refused for its query dtype
    # (checked before any launch; without a GPU the scratch lookup fails first)
    assert _call_static(s_fit, q_dtype=7) in (4, 6)


def _static_call(shape, dd, S, out, lse):
    import torch

    q_dtype = 1 if dd["q"].dtype == torch.bfloat16 else 0
    return b.lib.cvq_attend_static(
        ctypes.byref(shape), dd["q"].data_ptr(), q_dtype, dd["key_cb"].data_ptr(),
        dd["key_cb"].numel() // dd["key_cb"].shape[0], dd["key_codes"].data_ptr(),
        dd["val_codes"].data_ptr(), dd["seq_lens"].data_ptr(), dd["val_cb"].data_ptr(),
        dd["val_cb"].numel() // dd["val_cb"].shape[0], S, out.data_ptr(), lse.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
def test_static_calls_of_any_shape_in_any_order():
    import torch

    import compressed_attention_cvq_b200 as cvq
    from gpu_util import assert_close, run_oracle, to_device

    large = workloads.small(batch=1, n_q_heads=32, n_kv_heads=8, t_cap=4096, R=1, seed=202)
    small = workloads.small(batch=2, n_q_heads=8, n_kv_heads=2, t_cap=1500, R=2, q_dtype="bf16",
                            seq_lens=np.array([1500, 700], np.int32), seed=101, cb_std=0.7071)
    wide = workloads.small(batch=2, n_q_heads=8, n_kv_heads=2, t_cap=512, R=11,
                           seq_lens=np.array([512, 301], np.int32), seed=3,
                           cb_std=(1.0 / 11) ** 0.5, group_dim=64)
    cases = {"large": large, "small": small, "wide": wide}
    dev = {k: to_device(v) for k, v in cases.items()}
    ref = {k: run_oracle(v) for k, v in cases.items()}
    # large -> small -> large -> wide -> small: every smaller call after a larger one would
    # find the larger call's partial states where a shape-dependent counter offset puts it
    for name in ("large", "small", "large", "wide", "small"):
        d, dd = cases[name], dev[name]
        shape = cvq.shape_of(dd["q"], dd["key_codes"], d["rope_base"],
                             group_dim=d.get("group_dim", 8))
        S = cvq.suggest_splits(shape)
        # the caller-allocated path on a freshly zeroed workspace
        ws = cvq.workspace_alloc(shape, S, dd["q"].device)
        ref_out, ref_lse = cvq.attend_fused(shape, dd["q"], dd["key_cb"], dd["key_codes"],
                                            dd["val_codes"], dd["seq_lens"], dd["val_cb"], S,
                                            workspace=ws)
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        st = _static_call(shape, dd, S, out, lse)
        assert st == 0, (name, b.status_str(st))
        torch.cuda.synchronize()
        o, l = out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(l)), name
        # against the caller-allocated entry point, then against the oracle
        assert_close(o, l, ref_out.cpu().numpy().astype(np.float64),
                     ref_lse.cpu().numpy().astype(np.float64), out_tol=OUT_TOL, lse_rtol=LSE_RTOL)
        assert_close(o, l, *ref[name], out_tol=OUT_TOL, lse_rtol=LSE_RTOL)
    assert cvq.fault_status(clear=True) == 0
