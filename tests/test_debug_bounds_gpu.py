"""The debug build of the library (libcvq_debug.so: -DCVQ_DEBUG_BOUNDS) on small cases of
every decode kernel: the 4-head clustered kernel (R = 1 and 2), the plain kernel (one
query head per KV head, and the table form) and the 64-scalar-group kernel (R = 11).  Its
device-side range checks (code rows, codeword and bin indices, the exchange between the
CTAs of a pair, partial-state rows and arrival counters) must all pass -- the fault word
stays 0 -- and the results must still match the float64 oracle.  Runs in a child process
because the binding picks its library (CVQ_LIBRARY=debug) when it is first loaded."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import numpy as np, torch, sys
sys.path.insert(0, %(root)r); sys.path.insert(0, %(tests)r)
import workloads
import compressed_attention_cvq_b200 as cvq
from compressed_attention_cvq_b200 import _binding as b
from gpu_util import assert_close, run_gpu, run_oracle
assert b.LIB_PATH.endswith("libcvq_debug.so"), b.LIB_PATH
cases = [
    (dict(batch=2, n_q_heads=8, n_kv_heads=2, t_cap=1500, R=1, seq_lens=np.array([1500, 611], np.int32), seed=31), "gqa", 3),
    (dict(batch=2, n_q_heads=8, n_kv_heads=2, t_cap=900, R=2, q_dtype="bf16", cb_std=0.7071, seq_lens=np.array([900, 0], np.int32), seed=32), "gqa", 4),
    (dict(batch=1, n_q_heads=2, n_kv_heads=2, t_cap=700, R=2, seed=33), "gqa", 2),
    (dict(batch=1, n_q_heads=4, n_kv_heads=1, t_cap=700, R=1, seed=34), "table", 2),
    (dict(batch=2, n_q_heads=8, n_kv_heads=2, t_cap=512, R=11, cb_std=(1.0 / 11) ** 0.5, group_dim=64, seq_lens=np.array([512, 301], np.int32), seed=35), "gqa", 2),
]
for kw, form, S in cases:
    d = workloads.small(**kw)
    out, lse = run_gpu(d, form=form, n_splits=S)
    assert_close(out, lse, *run_oracle(d))
    word = cvq.fault_status(clear=True)
    assert word == 0, (kw, b.fault_names(word))
print("DEBUG_BOUNDS_OK")
"""


def test_debug_build_checks_pass_and_results_match_oracle():
    lib = os.path.join(ROOT, "compressed_attention_cvq_b200", "libcvq_debug.so")
    if not os.path.exists(lib):
        from compressed_attention_cvq_b200 import build as _build
        _build.build(debug_bounds=True)
    env = dict(os.environ, CVQ_LIBRARY="debug")
    code = CHILD % {"root": ROOT, "tests": os.path.join(ROOT, "tests")}
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "DEBUG_BOUNDS_OK" in r.stdout, r.stdout + r.stderr
