"""Register and spill budget of the decode kernels, read from ptxas (-Xptxas -v) on the
host: no GPU needed.  The designs depend on these budgets -- the 4-head kernel runs two
256-thread CTAs per SM at R = 1 (at most 128 registers a thread) and one 512-thread CTA at
R = 2, the 64-scalar-group kernel one 512-thread CTA -- and a spill puts local-memory
traffic into the per-token loop.  A source change that breaks a budget fails here before
it reaches a GPU."""
import functools
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@functools.lru_cache(maxsize=None)
def _ptxas_report(src):
    from compressed_attention_cvq_b200 import build as B

    try:
        nvcc = B.nvcc()
    except RuntimeError as e:
        pytest.skip(str(e))
    out = os.path.join("/tmp", f"cvq_res_{os.getpid()}_{os.path.basename(src)}.o")
    r = subprocess.run([nvcc, *B.ARCH, *B.FLAGS, "-Xptxas", "-v", "-c", src, "-o", out],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    if os.path.exists(out):
        os.remove(out)
    # entry name -> (registers, spill store bytes, spill load bytes)
    res, name = {}, None
    for line in r.stderr.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            name = m.group(1)
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and name:
            res[name] = [None, int(m.group(1)), int(m.group(2))]
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and name in res:
            res[name][0] = int(m.group(1))
    return res


@pytest.mark.parametrize("src,kernel,max_regs", [
    ("decode_gqa.cu", "decode_gqa4_kernelILi1E", 128),
    ("decode_gqa.cu", "decode_gqa4_kernelILi2E", 128),
    ("decode_wide.cu", "decode_wide_kernel", 128),
    # the naive attention's 4-head instance runs two 256-thread CTAs per SM
    ("naive_decode.cu", "naive_decode_kernelILi4E", 128),
])
def test_decode_kernels_fit_their_register_budget(src, kernel, max_regs):
    res = _ptxas_report(os.path.join(ROOT, "compressed_attention_cvq_b200", "csrc", src))
    hits = {k: v for k, v in res.items() if kernel in k}
    assert hits, f"no {kernel} entry in the ptxas report of {src}"
    for name, (regs, st, ld) in hits.items():
        assert regs is not None and regs <= max_regs, (name, regs)
        assert st == 0 and ld == 0, (name, st, ld)
